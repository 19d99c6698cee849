"""Pins for the CPU oracle: each check uses a formulation other than the oracle's own
(2-D slicing, subset enumeration, torch's dense attention with an explicit mask, finite
differences, torch autograd, hand-worked merges), so that a dropped term, a wrong index
or a transposed operand in the oracle fails at least one of them."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import pbsa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- geometry
def test_pages_cache_sizes_are_whole_frames():
    cfg = json.load(open(os.path.join(GOLDEN, "pages_config.json")))
    tf = cfg["frame_h"] * cfg["frame_w"]
    assert cfg["total_cache_size"] == cfg["local_cache_size"] + cfg["persistent_cache_size"]
    assert cfg["total_cache_size"] // tf == 12 and cfg["total_cache_size"] % tf == 0
    assert cfg["local_cache_size"] // tf == 6 and cfg["local_cache_size"] % tf == 0
    assert cfg["max_seq_len"] // tf == 21 and cfg["max_seq_len"] % tf == 0
    assert cfg["sparse_kv_block_size"] == [1, 8, 8]
    # 6 frames of 28 blocks -> 168 persistent slots, 168 local blocks, top-0.125 -> 21
    assert orc.n_slots(cfg["persistent_cache_size"], cfg["frame_h"], cfg["frame_w"]) == 168
    assert orc.topk_count(cfg["local_block_sparse_topk_ratio"], 168) == 21


def test_frame_blocks_partition_30x52():
    blocks = orc.frame_blocks(30, 52)
    assert len(blocks) == 28
    sizes = sorted(len(b) for b in blocks)
    assert sizes == sorted([64] * 18 + [32] * 3 + [48] * 6 + [24])
    allt = np.sort(np.concatenate(blocks))
    assert np.array_equal(allt, np.arange(1560))
    # block 6 is the right edge block of the first block row: x in [48, 52), y in [0, 8)
    ys, xs = np.divmod(blocks[6], 52)
    assert set(ys) == set(range(8)) and set(xs) == set(range(48, 52))
    # block 27 is the bottom-right corner: 6 x 4
    ys, xs = np.divmod(blocks[27], 52)
    assert set(ys) == set(range(24, 30)) and set(xs) == set(range(48, 52))


def test_pool_matches_2d_slicing():
    rng = np.random.default_rng(0)
    fh, fw, D, F = 12, 10, 5, 2
    x = rng.standard_normal((F, fh * fw, D))
    got = orc.pool_blocks(x, orc.frame_blocks(fh, fw))
    grid = x.reshape(F, fh, fw, D)
    want = []
    for f in range(F):
        for y0 in range(0, fh, 8):
            for x0 in range(0, fw, 8):
                want.append(grid[f, y0:y0 + 8, x0:x0 + 8].mean(axis=(0, 1)))
    assert np.allclose(got, np.stack(want), rtol=0, atol=1e-14)


def test_pool_constant_blocks_exact():
    fh, fw, D = 16, 12, 3
    blocks = orc.frame_blocks(fh, fw)
    x = np.zeros((1, fh * fw, D))
    for i, toks in enumerate(blocks):
        x[0, toks] = [i + 0.5, -i, 2.0 ** -i]
    got = orc.pool_blocks(x, blocks)
    for i in range(len(blocks)):
        assert list(got[i]) == [i + 0.5, -i, 2.0 ** -i]


# ---------------------------------------------------------------------------- selection
def test_topk_count_rule():
    assert orc.topk_count(0.125, 168) == 21
    assert orc.topk_count(0.25, 16) == 4
    assert orc.topk_count(0.0625, 84) == 6        # ceil(5.25)
    assert orc.topk_count(1e-9, 50) == 1          # at least one block
    assert orc.topk_count(1.0, 7) == 7
    assert orc.topk_count(0.125, 168, use_sparse=False) == 168
    assert orc.topk_count(0.5, 0) == 0


@pytest.mark.parametrize("seed", range(6))
def test_topk_equals_subset_enumeration(seed):
    rng = np.random.default_rng(seed)
    n, k = 8, 3
    s = np.round(rng.standard_normal(n), 1)   # coarse values -> frequent ties
    got = list(orc.select_topk(s, k))
    # the top-k set is the unique k-subset whose members all beat all non-members, where
    # "a beats b" is (s_a > s_b) or (s_a == s_b and a < b)
    beats = lambda a, b: s[a] > s[b] or (s[a] == s[b] and a < b)
    good = [c for c in itertools.combinations(range(n), k)
            if all(beats(a, b) for a in c for b in range(n) if b not in c)]
    assert len(good) == 1
    assert got == list(good[0])


def test_topk_ties_go_to_lower_index():
    s = np.array([1.0, 3.0, 2.0, 3.0, 2.0, 2.0])
    assert list(orc.select_topk(s, 1)) == [1]
    assert list(orc.select_topk(s, 2)) == [1, 3]
    assert list(orc.select_topk(s, 3)) == [1, 2, 3]
    assert list(orc.select_topk(s, 4)) == [1, 2, 3, 4]


def test_block_scores_closed_form():
    # query block = constant a*e0, key block j = constant c_j*e0 -> score a*c_j/sqrt(D)
    fh, fw, D = 8, 16, 4
    blocks = orc.frame_blocks(fh, fw)
    q = np.zeros((1, fh * fw, 1, D))
    k = np.zeros((1, 2 * fh * fw, 1, D))
    q[0, :, 0, 0] = 3.0
    c = [0.5, -1.0, 2.0, 0.25]
    for j in range(4):
        f, i = divmod(j, 2)
        k[0, f * fh * fw + blocks[i], 0, 0] = c[j]
    idx, sc = orc.select_blocks(q, k, fh, fw, ratio=0.5)
    assert np.allclose(sc[0, 0, 0], [3.0 * cj / 2.0 for cj in c], atol=0, rtol=1e-15)
    assert list(idx[0, 0, 0]) == [0, 2]


# ------------------------------------------------------------------------ tiny problem
def _tiny(seed=0, fh=12, fw=10, D=16, B=2, H=2, fq=2, fw_frames=3, S=5, filled=(0, 2, 3)):
    rng = np.random.default_rng(seed)
    tf = fh * fw
    q = rng.standard_normal((B, fq * tf, H, D)) * 0.7
    kw = rng.standard_normal((B, fw_frames * tf, H, D)) * 0.7
    vw = rng.standard_normal((B, fw_frames * tf, H, D))
    kp = np.zeros((B, H, S, 64, D))
    vp = np.zeros((B, H, S, 64, D))
    plen = np.zeros((B, H, S), dtype=np.int64)
    sizes = [len(t) for t in orc.frame_blocks(fh, fw)]
    for b in range(B):
        for h in range(H):
            for n, s in enumerate(filled):
                L = sizes[(n + b + h) % len(sizes)]
                plen[b, h, s] = L
                kp[b, h, s, :L] = rng.standard_normal((L, D)) * 0.7
                vp[b, h, s, :L] = rng.standard_normal((L, D))
    return dict(q=q, kw=kw, vw=vw, kp=kp, vp=vp, plen=plen, fh=fh, fw=fw)


def _dense_masked(t, idx, keep_persistent=True):
    """Dense formulation: all persistent rows + all window tokens as keys, with a boolean
    mask built from token coordinates, evaluated by torch's attention in fp64."""
    fh, fw = t["fh"], t["fw"]
    tf = fh * fw
    nbx = -(-fw // 8)
    nbf = -(-fh // 8) * nbx
    B, nq, H, D = t["q"].shape
    nw = t["kw"].shape[1]

    def blk(tok):  # block id of a token given by its position in a frame-major sequence
        f, n = divmod(tok, tf)
        y, x = divmod(n, fw)
        return f * nbf + (y // 8) * nbx + (x // 8)

    qblk = np.array([blk(i) for i in range(nq)])
    wblk = np.array([blk(i) for i in range(nw)])
    outs, lses, probs = {}, {}, {}
    for b in range(B):
        for h in range(H):
            prow = [t["kp"][b, h, s, :t["plen"][b, h, s]] for s in range(t["plen"].shape[2])]
            pv = [t["vp"][b, h, s, :t["plen"][b, h, s]] for s in range(t["plen"].shape[2])]
            kp = np.concatenate(prow) if keep_persistent else np.zeros((0, D))
            vp = np.concatenate(pv) if keep_persistent else np.zeros((0, D))
            keys = np.concatenate([kp, t["kw"][b, :, h]])
            vals = np.concatenate([vp, t["vw"][b, :, h]])
            mask = np.zeros((nq, len(keys)), dtype=bool)
            mask[:, :len(kp)] = True
            for i in range(nq):
                mask[i, len(kp):] = np.isin(wblk, idx[b, h, qblk[i]])
            qt = torch.tensor(t["q"][b, :, h])
            kt, vt, mt = torch.tensor(keys), torch.tensor(vals), torch.tensor(mask)
            o = torch.nn.functional.scaled_dot_product_attention(
                qt[None, None], kt[None, None], vt[None, None], attn_mask=mt[None, None])[0, 0]
            z = (qt @ kt.T) / math.sqrt(D)
            z = z.masked_fill(~mt, -math.inf)
            outs[b, h] = o.numpy()
            lses[b, h] = torch.logsumexp(z, dim=1).numpy()
            probs[b, h] = (torch.softmax(z, dim=1).numpy(), len(kp), wblk)
    return outs, lses, probs


def test_fwd_equals_dense_attention_when_all_selected_and_no_persistent():
    t = _tiny(filled=())
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=1.0)
    O, lse, mp, ml = orc.attn_fwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx,
                                  t["fh"], t["fw"])
    B, nq, H, D = t["q"].shape
    for b in range(B):
        for h in range(H):
            qt = torch.tensor(t["q"][b, :, h])[None, None]
            kt = torch.tensor(t["kw"][b, :, h])[None, None]
            vt = torch.tensor(t["vw"][b, :, h])[None, None]
            want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, 0].numpy()
            assert np.allclose(O[b, :, h], want, rtol=0, atol=1e-12)
            z = (qt[0, 0] @ kt[0, 0].T) / math.sqrt(D)
            assert np.allclose(lse[b, h], torch.logsumexp(z, 1).numpy(), rtol=0, atol=1e-12)
    assert np.allclose(mp, 0)


def test_fwd_equals_dense_attention_over_persistent_plus_window():
    t = _tiny()
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=1.0)
    O, lse, _, _ = orc.attn_fwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx,
                                t["fh"], t["fw"])
    outs, lses, _ = _dense_masked(t, idx)
    for (b, h), o in outs.items():
        assert np.allclose(O[b, :, h], o, rtol=0, atol=1e-12)
        assert np.allclose(lse[b, h], lses[b, h], rtol=0, atol=1e-12)


@pytest.mark.parametrize("ratio", [0.1, 0.25, 0.5])
def test_fwd_sparse_equals_masked_dense(ratio):
    t = _tiny(seed=3)
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=ratio)
    assert idx.shape[-1] == orc.topk_count(ratio, 3 * 4)
    O, lse, mp, ml = orc.attn_fwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx,
                                  t["fh"], t["fw"])
    outs, lses, probs = _dense_masked(t, idx)
    for (b, h), o in outs.items():
        assert np.allclose(O[b, :, h], o, rtol=0, atol=1e-12)
        assert np.allclose(lse[b, h], lses[b, h], rtol=0, atol=1e-12)
        # mass: column sums of the masked dense probabilities, grouped by owner block
        p, npers, wblk = probs[b, h]
        col = p.sum(axis=0)
        own = np.concatenate([np.full(int(t["plen"][b, h, s]), s)
                              for s in range(t["plen"].shape[2])])
        want_p = np.bincount(own, weights=col[:npers], minlength=t["plen"].shape[2])
        want_l = np.bincount(wblk, weights=col[npers:], minlength=ml.shape[-1])
        assert np.allclose(mp[b, h], want_p, rtol=0, atol=1e-12)
        assert np.allclose(ml[b, h], want_l, rtol=0, atol=1e-12)
        # every query row's probabilities sum to one
        assert math.isclose(mp[b, h].sum() + ml[b, h].sum(), t["q"].shape[1], rel_tol=1e-12)


def test_fwd_sample_restriction_matches_full_run():
    t = _tiny(seed=5)
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=0.25)
    O, lse, _, _ = orc.attn_fwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx,
                                t["fh"], t["fw"])
    Os, lses, _, _ = orc.attn_fwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx,
                                  t["fh"], t["fw"], heads=[(1, 0)], qblocks=[2, 5])
    blocks = orc.frame_blocks(t["fh"], t["fw"])
    tf = t["fh"] * t["fw"]
    for qb in (2, 5):
        toks = (qb // 4) * tf + blocks[qb % 4]
        assert np.array_equal(Os[1, toks, 0], O[1, toks, 0])
        assert np.array_equal(lses[1, 0, toks], lse[1, 0, toks])


# ----------------------------------------------------------------------------- backward
def _loss(t, idx, dO):
    O, _, _, _ = orc.attn_fwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx,
                              t["fh"], t["fw"])
    return float((O * dO).sum())


def test_bwd_matches_central_differences():
    t = _tiny(seed=7, B=1, H=1, D=8, fq=1, fw_frames=2, S=3, filled=(0, 2))
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=0.5)
    rng = np.random.default_rng(1)
    dO = rng.standard_normal(t["q"].shape)
    dQ, dKp, dVp, dKw, dVw = orc.attn_bwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"],
                                           t["vw"], idx, dO, t["fh"], t["fw"])
    eps = 1e-5
    checks = [("q", dQ), ("kw", dKw), ("vw", dVw), ("kp", dKp), ("vp", dVp)]
    for name, grad in checks:
        arr = t[name]
        flat = np.flatnonzero(np.ones(arr.shape))
        if name in ("kp", "vp"):  # only rows inside the slot lengths are inputs
            valid = np.zeros(arr.shape, dtype=bool)
            for s in range(arr.shape[2]):
                valid[:, :, s, :t["plen"][0, 0, s]] = True
            flat = np.flatnonzero(valid)
        pick = rng.choice(flat, size=12, replace=False)
        for f in pick:
            ix = np.unravel_index(f, arr.shape)
            old = arr[ix]
            arr[ix] = old + eps
            lp = _loss(t, idx, dO)
            arr[ix] = old - eps
            lm = _loss(t, idx, dO)
            arr[ix] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[ix]) < 1e-7 * max(1.0, abs(fd)), (name, ix, fd, grad[ix])


def test_bwd_matches_torch_autograd_masked_dense():
    t = _tiny(seed=11, B=1, H=2, D=16)
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=0.25)
    rng = np.random.default_rng(2)
    dO = rng.standard_normal(t["q"].shape)
    dQ, dKp, dVp, dKw, dVw = orc.attn_bwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"],
                                           t["vw"], idx, dO, t["fh"], t["fw"])
    fh, fw = t["fh"], t["fw"]
    tf, nbx = fh * fw, -(-fw // 8)
    nbf = -(-fh // 8) * nbx
    blk = lambda tok: (tok // tf) * nbf + ((tok % tf) // fw // 8) * nbx + ((tok % tf) % fw) // 8
    B, nq, H, D = t["q"].shape
    for h in range(H):
        q = torch.tensor(t["q"][0, :, h], requires_grad=True)
        kw = torch.tensor(t["kw"][0, :, h], requires_grad=True)
        vw = torch.tensor(t["vw"][0, :, h], requires_grad=True)
        kp = torch.tensor(t["kp"][0, h], requires_grad=True)
        vp = torch.tensor(t["vp"][0, h], requires_grad=True)
        S = kp.shape[0]
        rows = [(s, r) for s in range(S) for r in range(int(t["plen"][0, h, s]))]
        kpr = torch.stack([kp[s, r] for s, r in rows])
        vpr = torch.stack([vp[s, r] for s, r in rows])
        keys, vals = torch.cat([kpr, kw]), torch.cat([vpr, vw])
        mask = torch.zeros(nq, len(keys), dtype=torch.bool)
        mask[:, :len(rows)] = True
        wb = torch.tensor([blk(i) for i in range(kw.shape[0])])
        for i in range(nq):
            sel = torch.tensor(idx[0, h, blk(i)])
            mask[i, len(rows):] = torch.isin(wb, sel)
        z = (q @ keys.T / math.sqrt(D)).masked_fill(~mask, -math.inf)
        o = torch.softmax(z, dim=1) @ vals
        (o * torch.tensor(dO[0, :, h])).sum().backward()
        assert np.allclose(q.grad.numpy(), dQ[0, :, h], atol=1e-12)
        assert np.allclose(kw.grad.numpy(), dKw[0, :, h], atol=1e-12)
        assert np.allclose(vw.grad.numpy(), dVw[0, :, h], atol=1e-12)
        assert np.allclose(kp.grad.numpy(), dKp[0, h], atol=1e-12)
        assert np.allclose(vp.grad.numpy(), dVp[0, h], atol=1e-12)


def test_bwd_softmax_gradient_rows_sum_to_zero():
    # sum over keys of dS is zero for every row, so dQ is unchanged when every key is
    # shifted by the same vector
    t = _tiny(seed=13, B=1, H=1)
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=0.5)
    dO = np.random.default_rng(3).standard_normal(t["q"].shape)
    dQ = orc.attn_bwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx, dO,
                      t["fh"], t["fw"])[0]
    shift = np.random.default_rng(4).standard_normal(t["q"].shape[-1])
    t2 = dict(t)
    t2["kw"] = t["kw"] + shift
    kp = t["kp"].copy()
    for s in range(kp.shape[2]):
        kp[0, 0, s, :t["plen"][0, 0, s]] += shift
    t2["kp"] = kp
    dQ2 = orc.attn_bwd(t2["q"], t2["kp"], t2["vp"], t2["plen"], t2["kw"], t2["vw"], idx, dO,
                       t["fh"], t["fw"])[0]
    assert np.allclose(dQ, dQ2, atol=1e-10)


# ---------------------------------------------------------------------------- merge
def _merge_case(S, lens, scores, masses, n_evict_frames=1, fh=8, fw=12):
    """Persistent slots with given lengths/scores; a window of 2 frames of a 8x12 grid
    (blocks: 8x8 and 8x4) with given evicted-block masses."""
    D = 2
    B = H = 1
    tf = fh * fw
    kp = np.zeros((B, H, S, 64, D))
    vp = np.zeros((B, H, S, 64, D))
    plen = np.array(lens).reshape(1, 1, S)
    for s in range(S):
        kp[0, 0, s, :lens[s]] = 100 + s
        vp[0, 0, s, :lens[s]] = -100 - s
    psrc = np.where(plen > 0, 1000 + np.arange(S), -1)
    kw = np.arange(2 * tf * D, dtype=np.float64).reshape(1, 2 * tf, 1, D)
    vw = -kw
    ml = np.zeros((1, 1, 4))
    ml[0, 0, :len(masses)] = masses
    return orc.cache_update(kp, vp, plen, np.array(scores, float).reshape(1, 1, S), psrc,
                            kw, vw, ml, n_evict_frames, first_frame_global=7,
                            frame_h=fh, frame_w=fw), kw, vw


def test_merge_hand_example_full_cache():
    # slots: 0 (score 5), 1 empty, 2 (score 1); evicted blocks 0 (mass 3), 1 (mass 0.5).
    # Candidates 5, 1, 3, 0.5 -> keep slot 0, block 0, slot 2; block 0 takes empty slot 1.
    r, kw, _ = _merge_case(3, [64, 0, 32], [5.0, 0.0, 1.0], [3.0, 0.5])
    assert r["updates"][0][0] == [(1, 0)]
    assert list(r["pers_len"][0, 0]) == [64, 64, 32]
    assert list(r["pers_score"][0, 0]) == [5.0, 3.0, 1.0]
    # global id: frame 7 (oldest window frame), block 0 -> 7 * 2 + 0
    assert list(r["pers_src"][0, 0]) == [1000, 14, 1002]
    toks = orc.frame_blocks(8, 12)[0]
    assert np.array_equal(r["k_pers"][0, 0, 1, :64], kw[0, toks, 0])


def test_merge_hand_example_ties_keep_existing_slots_first():
    # all slots full with scores 2, 2, 1; evicted masses 2, 1 -> order s0, s1, b0, s2, b1;
    # keep s0, s1, b0; slot 2 is dropped and receives block 0.
    r, _, _ = _merge_case(3, [64, 64, 32], [2.0, 2.0, 1.0], [2.0, 1.0])
    assert r["updates"][0][0] == [(2, 0)]
    assert list(r["pers_len"][0, 0]) == [64, 64, 64]
    assert list(r["pers_src"][0, 0]) == [1000, 1001, 14]


def test_merge_hand_example_not_full_admits_everything():
    # one occupied slot (1); both evicted blocks admitted into empty slots 0 then 2.
    r, kw, vw = _merge_case(4, [0, 48, 0, 0], [0.0, 1.0, 0.0, 0.0], [0.1, 5.0])
    assert r["updates"][0][0] == [(0, 0), (2, 1)]
    assert list(r["pers_len"][0, 0]) == [64, 48, 32, 0]
    assert list(r["pers_score"][0, 0]) == [0.1, 1.0, 5.0, 0.0]
    assert list(r["pers_src"][0, 0]) == [14, 1001, 15, -1]
    toks = orc.frame_blocks(8, 12)[1]
    assert np.array_equal(r["v_pers"][0, 0, 2, :32], vw[0, toks, 0])
    assert np.all(r["v_pers"][0, 0, 2, 32:] == 0)


def test_merge_dropped_slot_not_refilled_ends_empty():
    # slots (3, 0.1); evicted blocks masses 9, 8 with only... capacity 2, 2 frames evicted:
    # candidates s0 3, s1 0.1, b0 9, b1 8, b2 0, b3 0 -> keep b0, b1; both slots dropped.
    r, _, _ = _merge_case(2, [64, 32], [3.0, 0.1], [9.0, 8.0, 0.0, 0.0], n_evict_frames=2)
    assert r["updates"][0][0] == [(0, 0), (1, 1)]
    assert list(r["pers_score"][0, 0]) == [9.0, 8.0]


@pytest.mark.parametrize("seed", range(8))
def test_merge_matches_rank_counting(seed):
    rng = np.random.default_rng(seed)
    S = 6
    lens = [int(x) for x in rng.choice([0, 32, 64], size=S)]
    scores = [float(np.round(rng.uniform(0, 3), 0)) if L else 0.0 for L in lens]
    masses = list(np.round(rng.uniform(0, 3, size=4), 0))
    r, _, _ = _merge_case(S, lens, scores, masses, n_evict_frames=2)
    occ = [s for s in range(S) if lens[s] > 0]
    cand = [scores[s] for s in occ] + masses
    # a candidate is kept iff fewer than S candidates come before it
    before = lambda a, b: cand[a] > cand[b] or (cand[a] == cand[b] and a < b)
    kept = [c for c in range(len(cand)) if sum(before(o, c) for o in range(len(cand))) < S]
    assert len(kept) == min(S, len(cand))
    kept_scores = sorted(cand[c] for c in kept)
    got = sorted(float(x) for s, x in enumerate(r["pers_score"][0, 0]) if r["pers_len"][0, 0, s] > 0)
    assert got == kept_scores
    assert (r["pers_len"][0, 0] > 0).sum() <= S
    for c in kept:   # kept slots did not move
        if c < len(occ):
            assert r["pers_src"][0, 0, occ[c]] == 1000 + occ[c]


def test_merge_hand_example_empty_slots_fill_before_dropped_ones():
    # slot 0 empty; slots 1, 2, 3 hold scores 1, 5, 0.2; evicted masses 4, 3.
    # Candidates s1 1, s2 5, s3 0.2, b0 4, b1 3 -> keep s2, b0, b1, s1; drop s3.
    # Free slots: empty slot 0 first, then dropped slot 3; blocks go there in id order.
    r, _, _ = _merge_case(4, [0, 64, 64, 32], [0.0, 1.0, 5.0, 0.2], [4.0, 3.0])
    assert r["updates"][0][0] == [(0, 0), (3, 1)]
    assert list(r["pers_len"][0, 0]) == [64, 64, 64, 32]
    assert list(r["pers_score"][0, 0]) == [4.0, 1.0, 5.0, 3.0]
    assert list(r["pers_src"][0, 0]) == [14, 1001, 1002, 15]


def test_dense_cache_mode_geometry():
    # page sizes: the dense window is the whole 18720-token cache (12 frames of 1560)
    assert orc.cache_geometry("dense", 18720, 9360, 9360, 30, 52) == (12, 0, True)
    assert orc.cache_geometry("sparse_forcing", 18720, 9360, 9360, 30, 52) == (6, 168, False)
    with pytest.raises(ValueError):
        orc.cache_geometry("paged", 18720, 9360, 9360, 30, 52)


def test_dense_cache_mode_forward_is_dense_attention_over_the_window():
    # dense mode = every window block selected and no persistent slots: plain attention
    t = _tiny(filled=())
    W, S, select_all = orc.cache_geometry("dense", t["kw"].shape[1], t["kw"].shape[1], 0,
                                          t["fh"], t["fw"])
    assert S == 0 and select_all
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio=0.25,
                               use_sparse=not select_all)
    nl = idx.shape[-1]
    assert (idx == np.arange(nl)).all()
    B, nq, H, D = t["q"].shape
    kp0 = np.zeros((B, H, 0, 64, D))
    O, lse, mp, ml = orc.attn_fwd(t["q"], kp0, kp0, np.zeros((B, H, 0), np.int64), t["kw"],
                                  t["vw"], idx, t["fh"], t["fw"])
    for b in range(B):
        for h in range(H):
            qt = torch.tensor(t["q"][b, :, h])[None, None]
            kt = torch.tensor(t["kw"][b, :, h])[None, None]
            vt = torch.tensor(t["vw"][b, :, h])[None, None]
            want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, 0].numpy()
            assert np.allclose(O[b, :, h], want, rtol=0, atol=1e-12)
    assert mp.size == 0


# ------------------------------------------------------------- slot count, multi-chunk
def test_n_slots_whole_frames_and_token_budget():
    # whole frames: frames x blocks per frame (16x16 has 4 blocks, 30x52 has 28)
    assert orc.n_slots(256, 16, 16) == 4
    assert orc.n_slots(512, 16, 16) == 8
    assert orc.n_slots(9360, 30, 52) == 168
    assert orc.n_slots(4680, 30, 52) == 84
    # otherwise the token budget in 64-row slots, rounded up
    assert orc.n_slots(64, 16, 16) == 1
    assert orc.n_slots(100, 16, 16) == 2
    assert orc.n_slots(129, 16, 16) == 3
    assert orc.n_slots(1000, 30, 52) == 16


@pytest.mark.parametrize("W,E,want", [(6, 3, [0, 3, 3, 3, 3]), (4, 1, [0, 0, 0, 1, 1, 1]),
                                      (5, 2, [0, 1, 2, 2, 2]), (2, 2, [2, 2, 2])])
def test_evict_count_hand_sequences(W, E, want):
    frames, got = 0, []
    for _ in want:
        frames += E            # the chunk joins the window
        assert frames <= W
        ev = orc.evict_count(frames, E, W)
        got.append(ev)
        frames -= ev
    assert got == want


def _hand_rollout_inputs():
    """Frames of 8x16 tokens (two 8x8 blocks), D = 4, one batch item and head.  Every query
    row is (2, 0, 0, 0); keys are zero except frame 2's block 1, whose tokens are
    (10, 0, 0, 0).  So a zero key scores logit 0, a hot key 2 * 10 / sqrt(4) = 10."""
    fh, fw, D = 8, 16, 4
    tf = fh * fw
    rng = np.random.default_rng(5)
    chunks = []
    for c in range(4):
        q = np.zeros((1, tf, 1, D))
        q[..., 0] = 2.0
        k = np.zeros((1, tf, 1, D))
        if c == 2:
            k[0, orc.frame_blocks(fh, fw)[1], 0, 0] = 10.0
        v = rng.standard_normal((1, tf, 1, D))
        chunks.append((q, k, v))
    return fh, fw, D, chunks


def test_decode_step_hand_rollout_fill_admit_and_turnover():
    """Window of 2 frames, 1-frame chunks, 2 persistent slots, ratio 0.5, values worked out
    by hand: uniform attention while every key is zero, then a hot block that takes almost
    all the probability and, two passes later, displaces the weaker slot."""
    fh, fw, D, chunks = _hand_rollout_inputs()
    st = orc.DecodeState.empty(1, 1, D, 2, fh, fw)
    outs = []
    for q, k, v in chunks:
        st, o = orc.decode_step(st, q, k, v, 0.5, 2, fh, fw)
        outs.append((st, o))
    Z = 192.0 + 64.0 * math.exp(10.0)
    a, hot = 8192.0 / Z, 8192.0 * math.exp(10.0) / Z     # per-pass mass of a cold / hot block
    # chunk 0: window [f0]; k = ceil(0.5 * 2) = 1 -> block 0 (tie to the lower id); every
    # row spreads over its 64 keys, so block 0 gets 128 rows x 1 and O = mean of its values
    st0, o0 = outs[0]
    assert o0["n_evict"] == 0 and o0["idx"].tolist() == [[[[0], [0]]]]
    assert np.allclose(o0["mass_local"][0, 0], [128.0, 0.0], rtol=0, atol=1e-12)
    vmean = chunks[0][2][0, orc.frame_blocks(fh, fw)[0], 0].mean(axis=0)
    assert np.allclose(o0["O"][0, :, 0], vmean, rtol=0, atol=1e-12)
    assert (st0.pers_len == 0).all()
    # chunk 1: window [f0, f1]; k = 2 -> blocks 0, 1 (all ties); 128 keys per row, 64 each;
    # accumulated f0 masses 192, 64; evict f0 into the empty cache in id order
    st1, o1 = outs[1]
    assert o1["idx"].tolist() == [[[[0, 1], [0, 1]]]]
    assert np.allclose(o1["mass_local"][0, 0], [64, 64, 0, 0], rtol=0, atol=1e-12)
    assert o1["n_evict"] == 1 and o1["updates"][0][0] == [(0, 0), (1, 1)]
    assert st1.pers_len.tolist() == [[[64, 64]]]
    assert np.allclose(st1.pers_score[0, 0], [192.0, 64.0], rtol=0, atol=1e-12)
    assert st1.pers_src.tolist() == [[[0, 1]]]
    assert np.allclose(st1.win_mass[0, 0], [0.0, 0.0]) and st1.first_frame_global == 1
    # chunk 2: window [f1, f2]; the hot block (id 3) scores 10, the rest 0 -> {0, 3};
    # keys per row: 128 slot rows + f1 block 0 (logit 0) + the hot block (logit 10)
    st2, o2 = outs[2]
    assert o2["idx"].tolist() == [[[[0, 3], [0, 3]]]]
    assert np.allclose(o2["mass_pers"][0, 0], [a, a], rtol=1e-12, atol=0)
    assert np.allclose(o2["mass_local"][0, 0], [a, 0.0, 0.0, hot], rtol=1e-12, atol=1e-15)
    assert o2["n_evict"] == 1 and o2["updates"][0][0] == []     # f1's blocks lose to both slots
    assert np.allclose(st2.pers_score[0, 0], [192 + a, 64 + a], rtol=1e-12, atol=0)
    assert np.allclose(st2.win_mass[0, 0], [0.0, hot], rtol=1e-12, atol=1e-15)
    # chunk 3: window [f2, f3]; the hot block is now id 1 -> {0, 1}; f2's block 1 has two
    # passes of mass (2 hot > 192 + 2a) and displaces slot 1 (64 + 2a)
    st3, o3 = outs[3]
    assert o3["idx"].tolist() == [[[[0, 1], [0, 1]]]]
    assert o3["n_evict"] == 1 and o3["updates"][0][0] == [(1, 1)]
    assert np.allclose(st3.pers_score[0, 0], [192 + 2 * a, 2 * hot], rtol=1e-12, atol=0)
    assert st3.pers_src.tolist() == [[[0, 2 * 2 + 1]]]     # global frame 2, block 1
    assert st3.pers_len.tolist() == [[[64, 64]]]
    assert (st3.k_pers[0, 0, 1, :, 0] == 10.0).all() and (st3.k_pers[0, 0, 1, :, 1:] == 0).all()
    assert st3.first_frame_global == 3 and st3.win_k.shape[1] == 128


# --------------------------------------------- [3,4,4] blocks (3 frames x 4 x 4 tokens)
def _block_of(pos, fh, fw, bt, bh, bw):
    """Block id of a token from its coordinates: position pos in a frame-major sequence ->
    frame, row, column -> (frame group, block row, block column)."""
    tf = fh * fw
    f, n = divmod(pos, tf)
    y, x = divmod(n, fw)
    nbx = -(-fw // bw)
    return (f // bt) * (-(-fh // bh) * nbx) + (y // bh) * nbx + x // bw


def test_frame_blocks_344_partition_30x52():
    blocks = orc.frame_blocks(30, 52, 4, 4, 3)
    assert len(blocks) == 8 * 13                       # 8 block rows (the last 2 high) x 13
    sizes = sorted(len(b) for b in blocks)
    assert sizes == sorted([48] * (7 * 13) + [24] * 13)
    allt = np.sort(np.concatenate(blocks))
    assert np.array_equal(allt, np.arange(3 * 1560))   # one group of 3 frames, each token once
    for i, b in enumerate(blocks):
        assert all(_block_of(p, 30, 52, 3, 4, 4) == i for p in b)
    # block 0: frames 0-2, rows 0-3, columns 0-3, frame by frame in raster order
    want = [t * 1560 + y * 52 + x for t in range(3) for y in range(4) for x in range(4)]
    assert blocks[0].tolist() == want
    assert orc.n_slots(9360, 30, 52, 4, 4, 3) == 2 * 104
    assert orc.n_slots(100, 8, 8, 4, 4, 3) == 3       # ceil(100 / 48)
    assert orc.slot_capacity(4, 4, 3) == 48


def test_pool_344_matches_3d_slicing():
    rng = np.random.default_rng(8)
    fh, fw, D, G = 10, 8, 3, 2                          # 2 groups of 3 frames
    x = rng.standard_normal((G * 3 * fh * fw, D))
    got = orc.pool_blocks(x.reshape(G, 3 * fh * fw, D), orc.frame_blocks(fh, fw, 4, 4, 3))
    grid = x.reshape(G, 3, fh, fw, D)
    want = [grid[g, :, y0:y0 + 4, x0:x0 + 4].mean(axis=(0, 1, 2))
            for g in range(G) for y0 in range(0, fh, 4) for x0 in range(0, fw, 4)]
    assert np.allclose(got, np.stack(want), rtol=0, atol=1e-14)


def _tiny344(seed, B=1, H=2, D=8, fh=6, fw=8, q_groups=1, w_groups=2, S=4, filled=(0, 1, 3)):
    rng = np.random.default_rng(seed)
    tg = 3 * fh * fw
    t = dict(q=rng.standard_normal((B, q_groups * tg, H, D)) * 0.7,
             kw=rng.standard_normal((B, w_groups * tg, H, D)) * 0.7,
             vw=rng.standard_normal((B, w_groups * tg, H, D)),
             kp=np.zeros((B, H, S, 64, D)), vp=np.zeros((B, H, S, 64, D)),
             plen=np.zeros((B, H, S), np.int64), fh=fh, fw=fw)
    sizes = [len(b) for b in orc.frame_blocks(fh, fw, 4, 4, 3)]     # 48 and 24 at 6x8
    for b in range(B):
        for h in range(H):
            for n, s in enumerate(filled):
                L = sizes[(n + h) % len(sizes)]
                t["plen"][b, h, s] = L
                t["kp"][b, h, s, :L] = rng.standard_normal((L, D)) * 0.7
                t["vp"][b, h, s, :L] = rng.standard_normal((L, D))
    return t


def _masked_dense_344(t, idx, b, h, requires_grad=False):
    """Keys = every persistent row then every window token; a window token is visible to a
    query token iff the key's block (from its coordinates) is in the query's block list."""
    fh, fw = t["fh"], t["fw"]
    nq, nw = t["q"].shape[1], t["kw"].shape[1]
    T = lambda a: torch.tensor(a, requires_grad=requires_grad)
    q, kw, vw, kp, vp = T(t["q"][b, :, h]), T(t["kw"][b, :, h]), T(t["vw"][b, :, h]), \
        T(t["kp"][b, h]), T(t["vp"][b, h])
    rows = [(s, r) for s in range(kp.shape[0]) for r in range(int(t["plen"][b, h, s]))]
    keys = torch.cat([torch.stack([kp[s, r] for s, r in rows]), kw])
    vals = torch.cat([torch.stack([vp[s, r] for s, r in rows]), vw])
    wb = np.array([_block_of(p, fh, fw, 3, 4, 4) for p in range(nw)])
    mask = np.zeros((nq, len(keys)), dtype=bool)
    mask[:, :len(rows)] = True
    for i in range(nq):
        mask[i, len(rows):] = np.isin(wb, idx[b, h, _block_of(i, fh, fw, 3, 4, 4)])
    z = (q @ keys.T / math.sqrt(q.shape[1])).masked_fill(~torch.tensor(mask), -math.inf)
    p = torch.softmax(z, dim=1)
    return dict(o=p @ vals, lse=torch.logsumexp(z, 1), p=p, npers=len(rows), wb=wb, rows=rows,
                leaves=(q, kw, vw, kp, vp))


@pytest.mark.parametrize("ratio", [0.25, 0.5])
def test_fwd_344_equals_masked_dense(ratio):
    t = _tiny344(seed=21)
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], ratio, bh=4, bw=4, bt=3)
    assert idx.shape[2] == 4 and idx.shape[-1] == orc.topk_count(ratio, 2 * 4)
    O, lse, mp, ml = orc.attn_fwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"], idx,
                                  t["fh"], t["fw"], 4, 4, bt=3)
    for h in range(t["q"].shape[2]):
        r = _masked_dense_344(t, idx, 0, h)
        assert np.allclose(O[0, :, h], r["o"].numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse[0, h], r["lse"].numpy(), rtol=0, atol=1e-12)
        col = r["p"].numpy().sum(axis=0)
        own = np.array([s for s, _ in r["rows"]])
        assert np.allclose(mp[0, h], np.bincount(own, col[:r["npers"]], t["plen"].shape[2]), atol=1e-12)
        assert np.allclose(ml[0, h], np.bincount(r["wb"], col[r["npers"]:], 8), atol=1e-12)


def test_bwd_344_matches_torch_autograd_masked_dense():
    t = _tiny344(seed=22, H=1)
    idx, _ = orc.select_blocks(t["q"], t["kw"], t["fh"], t["fw"], 0.5, bh=4, bw=4, bt=3)
    dO = np.random.default_rng(9).standard_normal(t["q"].shape)
    dQ, dKp, dVp, dKw, dVw = orc.attn_bwd(t["q"], t["kp"], t["vp"], t["plen"], t["kw"], t["vw"],
                                           idx, dO, t["fh"], t["fw"], 4, 4, bt=3)
    r = _masked_dense_344(t, idx, 0, 0, requires_grad=True)
    (r["o"] * torch.tensor(dO[0, :, 0])).sum().backward()
    q, kw, vw, kp, vp = r["leaves"]
    for got, want in [(q, dQ[0, :, 0]), (kw, dKw[0, :, 0]), (vw, dVw[0, :, 0]), (kp, dKp[0, 0]),
                      (vp, dVp[0, 0])]:
        assert np.allclose(got.grad.numpy(), want, rtol=0, atol=1e-12)


def test_merge_344_hand_example():
    # frames of 4x8 tokens: a group of 3 frames has two 3x4x4 blocks of 48 tokens.  Window of
    # 2 groups (6 frames), its oldest frame being global frame 6 (group 2).  Slots: 0 holds a
    # block with score 5, slot 1 is empty.  Evicting one group (3 frames) with masses 3 and
    # 0.5: candidates 5, 3, 0.5 -> block 0 enters slot 1 with source 2 * 2 + 0 = 4.
    fh, fw, D = 4, 8, 2
    tg = 3 * fh * fw
    kp = np.zeros((1, 1, 2, 64, D))
    kp[0, 0, 0, :48] = 1.0
    plen = np.array([[[48, 0]]])
    kw = np.arange(2 * tg * D, dtype=np.float64).reshape(1, 2 * tg, 1, D)
    ml = np.array([[[3.0, 0.5, 0.0, 0.0]]])
    r = orc.cache_update(kp, kp, plen, np.array([[[5.0, 0.0]]]), np.array([[[77, -1]]]), kw, -kw,
                         ml, 3, 6, fh, fw, 4, 4, bt=3)
    assert r["updates"][0][0] == [(1, 0)]
    assert r["pers_len"].tolist() == [[[48, 48]]]
    assert r["pers_src"].tolist() == [[[77, 4]]]
    toks = [t * 32 + y * 8 + x for t in range(3) for y in range(4) for x in range(4)]
    assert np.array_equal(r["k_pers"][0, 0, 1, :48], kw[0, toks, 0])
    assert np.all(r["k_pers"][0, 0, 1, 48:] == 0)
    with pytest.raises(ValueError):
        orc.cache_update(kp, kp, plen, np.zeros((1, 1, 2)), np.zeros((1, 1, 2), int), kw, kw, ml,
                         2, 6, fh, fw, 4, 4, bt=3)


# ------------------------------------------------------------------------------ sink
def test_sink_slot_counts():
    assert orc.sink_slots(1, 30, 52) == 28
    assert orc.sink_slots(2, 16, 16) == 8
    assert orc.sink_slots(3, 30, 52, 4, 4, 3) == 104
    assert orc.sink_slots(0, 30, 52) == 0
    with pytest.raises(ValueError):
        orc.sink_slots(2, 30, 52, 4, 4, 3)


def test_merge_never_touches_sink_slots():
    # Without a sink, the candidates 0.01, 5, 1 (slots) and 3, 0.5 (blocks) keep slot 1,
    # block 0 and slot 2: slot 0 is dropped and receives block 0.
    r, _, _ = _merge_case(3, [64, 64, 32], [0.01, 5.0, 1.0], [3.0, 0.5])
    assert r["updates"][0][0] == [(0, 0)]
    # With slot 0 a sink slot, 2 ordinary slots compete: 5, 1, 3, 0.5 keep slot 1 and
    # block 0; slot 2 is dropped and receives block 0.  The sink slot stays although every
    # candidate beats it.
    fh, fw, D = 8, 12, 2
    kp = np.zeros((1, 1, 3, 64, D))
    kp[0, 0, 0, :64] = 7.0
    plen = np.array([[[64, 64, 32]]])
    kw = np.arange(2 * 96 * D, dtype=np.float64).reshape(1, 2 * 96, 1, D)
    ml = np.zeros((1, 1, 4))
    ml[0, 0, :2] = [3.0, 0.5]
    r = orc.cache_update(kp, kp, plen, np.array([[[0.01, 5.0, 1.0]]]), np.array([[[0, 11, 12]]]),
                         kw, kw, ml, 1, 2, fh, fw, n_sink=1)
    assert r["updates"][0][0] == [(2, 0)]
    assert r["pers_src"].tolist() == [[[0, 11, 2 * 2 + 0]]]
    assert r["pers_score"].tolist() == [[[0.01, 5.0, 3.0]]]
    assert (r["k_pers"][0, 0, 0, :64] == 7.0).all()


def test_decode_step_with_a_sink_frame_hand_rollout():
    """Frames of 8x8 tokens (one block), D = 4, 2-frame chunks, a 4-frame window, 2 ordinary
    slots and a 1-frame sink, ratio 1 (every window block).  Queries are (2, 0, 0, 0); the
    sink frame's keys are (-10, 0, 0, 0) (logit -10), every other key is zero (logit 0)."""
    fh = fw = 8
    D, tf = 4, 64
    rng = np.random.default_rng(4)
    chunks = []
    for c in range(3):
        q = np.zeros((1, 2 * tf, 1, D))
        q[..., 0] = 2.0
        k = np.zeros((1, 2 * tf, 1, D))
        if c == 0:
            k[0, :tf, 0, 0] = -10.0          # global frame 0: the sink
        chunks.append((q, k, rng.standard_normal((1, 2 * tf, 1, D))))
    n_sink = orc.sink_slots(1, fh, fw)
    st = orc.DecodeState.empty(1, 1, D, n_sink + 2, fh, fw)
    res = []
    for q, k, v in chunks:
        st, o = orc.decode_step(st, q, k, v, 1.0, 4, fh, fw, sink_frames=1)
        res.append((st, o))
    e = math.exp(-10.0)
    # chunk 0: frame 0 goes to sink slot 0, frame 1 into the window; 128 query rows over
    # 64 sink keys (weight e^-10) and 64 window keys (weight 1)
    st0, o0 = res[0]
    assert st0.win_k.shape[1] == tf and st0.first_frame_global == 1 and o0["n_evict"] == 0
    assert st0.pers_len.tolist() == [[[64, 0, 0]]] and st0.pers_src.tolist() == [[[0, -1, -1]]]
    assert np.allclose(o0["mass_pers"][0, 0, 0], 128 * e / (1 + e), rtol=1e-12)
    assert np.allclose(o0["mass_local"][0, 0], [128 / (1 + e)], rtol=1e-12)
    # chunk 1: window [f1, f2, f3]; Z = 64 e + 192; then f1 leaves and takes ordinary slot 1
    Z1 = 64 * e + 192
    st1, o1 = res[1]
    assert np.allclose(o1["mass_local"][0, 0], [8192 / Z1] * 3, rtol=1e-12)
    assert o1["n_evict"] == 1 and o1["updates"][0][0] == [(1, 0)]
    assert st1.pers_src.tolist() == [[[0, 1, -1]]]
    assert np.allclose(st1.pers_score[0, 0, 1], 128 / (1 + e) + 8192 / Z1, rtol=1e-12)
    # chunk 2: window [f2 .. f5]; Z = 64 e + 320; f2 and f3 leave with equal masses; the one
    # free ordinary slot goes to f2 (the lower id) and f3 is dropped; the sink slot, whose
    # mass is the smallest of all, is no candidate and stays
    Z2 = 64 * e + 320
    st2, o2 = res[2]
    assert o2["n_evict"] == 2 and o2["updates"][0][0] == [(2, 0)]
    assert st2.pers_src.tolist() == [[[0, 1, 2]]] and st2.pers_len.tolist() == [[[64, 64, 64]]]
    assert np.allclose(st2.pers_score[0, 0, 2], 8192 / Z1 + 8192 / Z2, rtol=1e-12)
    assert st2.pers_score[0, 0, 0] < 1e-2 < st2.pers_score[0, 0, 2]
    assert (st2.k_pers[0, 0, 0, :, 0] == -10.0).all()
    assert st2.first_frame_global == 4 and st2.win_k.shape[1] == 2 * tf
