"""Rollout with memory updates (decode geometry, 20 chunks of 3 frames, fresh K/V each
chunk, empty persistent cache at the start): every step runs selection, the forward with
block mass, the window slide and the persistent merge on the GPU through the C ABI
(SparseForcingAttention wrapper), and the oracle replays that step from the GPU's state at
the start of the step.  Index lists, outputs, masses, merge decisions and cache contents
are compared step by step.  One head keeps the oracle's time low; heads are independent."""
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200.attention import SparseForcingAttention
from block_sparse_attention_35_b200.synth import WORKLOADS, rollout_chunk, rollout_chunk_hot
from oracle import pbsa_oracle as orc
from tests.harness import (LSE_ABS, MASS_ABS, MASS_REL, assert_close_bf16, check_topk, f64,
                           ring_to_window)

pytestmark = pytest.mark.gpu


def _logical_mass(ml_phys, ring_head, local_frames, W, nbf, bt=1):
    Wg = W // bt
    out = np.zeros(ml_phys.shape[:2] + (local_frames // bt * nbf,))
    for lid in range(local_frames // bt * nbf):
        out[:, :, lid] = ml_phys[:, :, ((ring_head // bt + lid // nbf) % Wg) * nbf + lid % nbf]
    return out


def _state_from_gpu(a, W, tf, nbf):
    """The oracle's DecodeState holding the wrapper's current caches (window in logical
    order, masses by logical block)."""
    lf, rh = a.local_frames, a.ring_head
    win = lambda t: (f64(ring_to_window(t.cpu(), rh, lf, W, tf)) if lf else
                     np.zeros((t.shape[0], 0) + tuple(t.shape[2:])))
    return orc.DecodeState(
        win(a.k_local), win(a.v_local),
        _logical_mass(a.mass_local.cpu().double().numpy(), rh, lf, W, nbf, a.bt),
        f64(a.k_pers), f64(a.v_pers), a.pers_len.cpu().numpy(),
        a.pers_score.cpu().double().numpy(), a.pers_src.cpu().numpy(), a.first_frame_global)


def _run_rollout(wl, dev, chunks, chunk_fn, sink_frames=0):
    a = SparseForcingAttention(wl.B, wl.H, wl.D, wl.frame_h, wl.frame_w, wl.total_cache_size,
                               wl.local_cache_size, wl.persistent_cache_size,
                               sparse_kv_block_size=wl.block, max_seq_len=wl.max_seq_len,
                               local_block_sparse_topk_ratio=wl.topk_ratio,
                               chunk_frames=wl.q_frames, sink_frames=sink_frames, device=dev)
    W, tf, nbf, S = a.W, a.tf, a.nbf, a.S
    bt, bh, bw = wl.block
    n_sink = a.n_sink
    exact_frac, admitted = [], []
    for step in range(chunks):
        q, k, v = chunk_fn(step)
        st0 = _state_from_gpu(a, W, tf, nbf)          # state before the chunk joins
        a.append(k.to(dev), v.to(dev))
        lf, rh = a.local_frames, a.ring_head
        a(q.to(dev), accumulate_mass=True)
        torch.cuda.synchronize()
        assert int(a.status.item()) == 0
        idx = a.idx.cpu().numpy()
        # ---- the oracle's step on the same state, with the GPU's selection (near-ties may
        # legitimately differ; the selection itself is checked against the oracle's scores)
        st1, o = orc.decode_step(st0, f64(q), f64(k), f64(v), wl.topk_ratio, W, wl.frame_h,
                                 wl.frame_w, idx=idx[..., :P_k(a, lf)], bh=bh, bw=bw, bt=bt,
                                 sink_frames=sink_frames)
        appended = orc.append_frames(st0, f64(k), f64(v), sink_frames, wl.frame_h, wl.frame_w,
                                     bh, bw, bt)
        kwin, vwin = appended.win_k, appended.win_v
        assert np.array_equal(a.pers_len.cpu().numpy(), appended.pers_len)
        assert np.array_equal(f64(a.k_pers), appended.k_pers)
        kk = P_k(a, lf)
        if kk:
            _, sc_o = orc.select_blocks(f64(q), kwin, wl.frame_h, wl.frame_w, wl.topk_ratio,
                                        bh=bh, bw=bw, bt=bt)
            exact_frac.append(check_topk(idx[..., :kk], a.cnt.cpu().numpy(), sc_o, kk))
        assert_close_bf16(f64(a.out), o["O"], f"step {step} out")
        assert np.abs(a.lse.cpu().numpy() - o["lse"]).max() <= LSE_ABS
        ps1 = a.pers_score.cpu().double().numpy()
        ml1 = _logical_mass(a.mass_local.cpu().double().numpy(), rh, lf, W, nbf, bt)
        assert np.allclose(ps1, o["pers_score_before_merge"], rtol=MASS_REL, atol=MASS_ABS)
        assert np.allclose(ml1, o["win_mass_before_merge"], rtol=MASS_REL, atol=MASS_ABS)
        # ---- slide + merge: the eviction count is the oracle's
        n_ev = o["n_evict"]
        assert a.slide() == n_ev
        torch.cuda.synchronize()
        nup = [int(x) for x in a.n_upd.cpu().numpy().ravel()] if n_ev else [0]
        if n_ev:
            ups = [tuple(x) for x in a.upd[0, 0, :nup[0]].cpu().numpy()]
            # decisions on the GPU's own masses must match the oracle's merge exactly
            r = orc.cache_update(appended.k_pers, appended.v_pers, appended.pers_len, ps1,
                                 appended.pers_src, kwin, vwin, ml1, n_ev,
                                 appended.first_frame_global, wl.frame_h, wl.frame_w, bh, bw, bt,
                                 n_sink)
            assert ups == r["updates"][0][0], f"step {step}"
            assert np.array_equal(a.pers_len.cpu().numpy(), r["pers_len"])
            assert np.array_equal(a.pers_src.cpu().numpy(), r["pers_src"])
            assert np.array_equal(f64(a.k_pers), r["k_pers"])
            assert np.array_equal(f64(a.v_pers), r["v_pers"])
            # and the oracle's own step (its masses) decides the same wherever the keep/drop
            # margin exceeds 1e-3
            cand = [o["pers_score_before_merge"][0, 0, s] for s in range(n_sink, S)
                    if appended.pers_len[0, 0, s] > 0]
            cand += list(o["win_mass_before_merge"][0, 0, :n_ev // bt * nbf])
            srt = sorted(cand, reverse=True)
            Sm = S - n_sink
            margin = (srt[Sm - 1] - srt[Sm]) if len(srt) > Sm else np.inf
            if margin > 1e-3:
                assert o["updates"][0][0] == ups, f"step {step}: decision differs at margin {margin}"
                assert np.array_equal(st1.pers_len, a.pers_len.cpu().numpy())
        assert a.local_frames == st1.win_k.shape[1] // tf
        assert a.first_frame_global == st1.first_frame_global
        admitted.append(nup[0])
    return a, exact_frac, admitted


def P_k(a, local_frames):
    from block_sparse_attention_35_b200 import pbsa as P
    return P.pbsa_topk_count(a.cfg, local_frames)


def test_rollout_twenty_chunks(cuda_dev):
    wl = dataclasses.replace(WORKLOADS["rollout"], H=1)
    a, exact_frac, admitted = _run_rollout(wl, cuda_dev, wl.chunks, lambda s: rollout_chunk(wl, s))
    # the persistent cache filled up (chunks 1 and 2 admit 84 blocks each).  Slots keep
    # accumulating mass while cached, so with stationary synthetic queries later evicted
    # blocks (two chunks of mass) rank below the slots: every later step checks a merge
    # that admits nothing, which the decisions above verified against the oracle.
    assert int((a.pers_len > 0).sum().item()) == a.S
    assert sum(admitted) >= a.S
    print(f"rollout: exact top-k fraction per step {np.round(exact_frac, 3).tolist()}, "
          f"admissions {admitted}")


def test_rollout_hot_blocks_turn_the_cache_over(cuda_dev):
    """Rollout in which every chunk carries a few "hot" key blocks aligned with the queries:
    they gather most of the attention mass, so evicted hot blocks keep displacing slots
    after the cache is full (turnover), and every merge is checked against the oracle."""
    wl = dataclasses.replace(WORKLOADS["rollout"], H=1, chunks=8)
    a, _, admitted = _run_rollout(wl, cuda_dev, wl.chunks, lambda s: rollout_chunk_hot(wl, s))
    full_at = next(i for i in range(len(admitted)) if sum(admitted[:i + 1]) >= a.S)
    assert sum(admitted[full_at + 1:]) > 0, f"no admissions after the cache filled: {admitted}"
    print(f"hot rollout: admissions {admitted}")


def test_rollout_with_a_sink_frame(cuda_dev):
    """Decode geometry (one head), the first frame of the sequence as the sink: its 28
    blocks live in sink slots from chunk 0 on, are attended by every query, and no merge
    touches them; 6 chunks, every step replayed by the oracle."""
    wl = dataclasses.replace(WORKLOADS["rollout"], H=1, chunks=6)
    a, _, admitted = _run_rollout(wl, cuda_dev, wl.chunks, lambda s: rollout_chunk_hot(wl, s),
                                  sink_frames=1)
    assert a.n_sink == 28
    assert (a.pers_len[0, 0, :28] > 0).all() and (a.pers_src[0, 0, :28].cpu() == torch.arange(28)).all()
    assert sum(admitted) > 0
