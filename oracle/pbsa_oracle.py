"""Plain fp64 CPU oracle for Persistent Block-Sparse Attention (PBSA).

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline
arm of ``bench.py`` may import this module.  The library (``block_sparse_attention_35_b200``)
never imports it and has no CPU fallback.

Sources (no page prints the method's equations; the rules below are the plainest
reading of what the pages state):

* "Sparse Forcing: Native Trainable Sparse Attention for Real-time Autoregressive
  Diffusion Video Generation" (pith.science), abstract: attention over a persistent set of
  salient blocks kept in the KV cache ("compress, preserve, and update") plus a
  dynamically selected neighbourhood inside each sliding local window; PBSA accelerates
  the sparse attention and the memory updates.
* Same page, algorithm fragment in the reference list (training loop): the t=0 pass
  applies PBSA with top-k and updates P (persistent) and L (local); denoising passes
  apply PBSA with top-k only.
* Project page (boxunxu.top/SparseForcing), usage snippet of ``SparseForcingAttention``:
  ``total_cache_size``, ``local_cache_size``, ``persistent_cache_size``,
  ``sparse_kv_block_size=[1, 8, 8]``, ``max_seq_len``, ``use_local_block_sparse_attn``,
  ``local_block_sparse_topk_ratio`` and the call ``attn(query, key_persistent,
  value_persistent, key_local, value_local)``; kernel features: local + persistent
  block-sparse attention, learned top-k, full gradient support.

Readings taken where the pages are silent (each is a choice, listed in the design notes):
block score = mean-pooled query block . mean-pooled key block / sqrt(D), ties to the lower
block index; k = clamp(ceil(ratio * N_L), 1, N_L); ragged edge blocks pool and attend over
their valid tokens only; block mass = sum over query rows of the softmax probability that
falls on the block, accumulated while the block is cached; eviction merges the evicted
frames' blocks into the persistent set by mass, keeping the highest-mass blocks.

Everything is float64.  bf16 inputs are converted exactly.  Loops run over (batch, head,
query block) so that each step can be checked against the readings by eye.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["frame_blocks", "topk_count", "pool_blocks", "block_scores", "select_topk",
           "select_blocks", "attend_rows", "attn_fwd", "cache_update", "attn_bwd",
           "slot_capacity", "n_slots", "sink_slots", "evict_count", "append_frames",
           "DecodeState", "decode_step"]


# ---------------------------------------------------------------------------------------
# Geometry (project page, usage snippet: sparse_kv_block_size=[1, 8, 8]; the comparison
# table's "[3,4,4] block size" rows: blocks of 3 frames x 4 x 4 tokens)
# ---------------------------------------------------------------------------------------
def frame_blocks(frame_h: int, frame_w: int, bh: int = 8, bw: int = 8, bt: int = 1):
    """Token indices of each bt x bh x bw block of one group of bt consecutive frames.

    Tokens of a frame are numbered in raster order (n = y * frame_w + x) and the frames of
    a group follow one another, so token (t, y, x) of the group is t * frame_h * frame_w +
    y * frame_w + x.  Blocks are numbered row of blocks first: id = by * ceil(frame_w / bw)
    + bx; every block spans all bt frames of the group.  Edge blocks are clipped to the
    frame (reading: ragged blocks hold only their valid tokens).  Inside a block tokens are
    listed frame by frame, each frame in raster order; this is also the row order of a
    block copied into a persistent slot.  With bt = 1 a group is one frame.
    """
    tf = frame_h * frame_w
    out = []
    for y0 in range(0, frame_h, bh):
        for x0 in range(0, frame_w, bw):
            toks = [t * tf + y * frame_w + x
                    for t in range(bt)
                    for y in range(y0, min(y0 + bh, frame_h))
                    for x in range(x0, min(x0 + bw, frame_w))]
            out.append(np.asarray(toks, dtype=np.int64))
    return out


def slot_capacity(bh: int = 8, bw: int = 8, bt: int = 1) -> int:
    """Tokens of one full block, which one persistent slot holds."""
    return bt * bh * bw


def n_slots(persistent_cache_size: int, frame_h: int, frame_w: int, bh=8, bw=8, bt=1) -> int:
    """Persistent capacity in blocks (reading: the blocks of the whole frame groups the token
    budget holds; otherwise the budget in full blocks, rounded up)."""
    tg = bt * frame_h * frame_w
    if persistent_cache_size % tg == 0:
        return persistent_cache_size // tg * len(frame_blocks(frame_h, frame_w, bh, bw, bt))
    return -(-persistent_cache_size // (bt * bh * bw))


def sink_slots(sink_frames: int, frame_h: int, frame_w: int, bh=8, bw=8, bt=1) -> int:
    """Persistent slots reserved for the sink (project page, kernel features: "local, sink,
    and learned top-k" sparsity patterns).  Reading: the sink is the first sink_frames
    frames of the sequence (a multiple of bt); each of their blocks keeps one slot of its
    own at the front of the slot store, in addition to the slots of persistent_cache_size,
    so that every query attends to them for the whole sequence."""
    if sink_frames % bt:
        raise ValueError("sink_frames must be a multiple of the block's frame count")
    return sink_frames // bt * len(frame_blocks(frame_h, frame_w, bh, bw, bt))


def cache_geometry(kv_cache_mode: str, total_cache_size: int, local_cache_size: int,
                   persistent_cache_size: int, frame_h: int, frame_w: int, bh=8, bw=8, bt=1):
    """(window frames W, persistent slots S, every window block attended?) of a cache mode.

    kv_cache_mode="sparse_forcing" (project page, constructor default): a window of
    local_cache_size tokens plus the persistent slots.  "dense" (reading: the plain cache
    the pages compare Sparse Forcing with; the page names no other mode): one window of
    total_cache_size tokens, no persistent slots, every block attended, eviction drops.
    """
    tf = frame_h * frame_w
    if kv_cache_mode == "dense":
        return total_cache_size // tf, 0, True
    if kv_cache_mode != "sparse_forcing":
        raise ValueError(kv_cache_mode)
    return local_cache_size // tf, n_slots(persistent_cache_size, frame_h, frame_w, bh, bw, bt), False


# ---------------------------------------------------------------------------------------
# Block selection (project page: learned top-k selection, local_block_sparse_topk_ratio;
# pith abstract: "dynamically selected local neighborhood")
# ---------------------------------------------------------------------------------------
def topk_count(ratio: float, n_local: int, use_sparse: bool = True) -> int:
    """Number of local blocks each query block attends to.

    With use_local_block_sparse_attn off every local block is used.  Otherwise
    k = ceil(ratio * N_L) clamped to [1, N_L] (reading: the pages give only the ratio).
    """
    if n_local <= 0:
        return 0
    if not use_sparse:
        return n_local
    return min(n_local, max(1, math.ceil(ratio * n_local)))


def pool_blocks(x_frames: np.ndarray, blocks) -> np.ndarray:
    """Mean over the valid tokens of every block.

    x_frames: [F, T_f, D] (one batch item and head, frames oldest first).
    Returns [F * NB_f, D]; block id = frame * NB_f + block-in-frame.
    """
    x = np.asarray(x_frames, dtype=np.float64)
    rows = []
    for f in range(x.shape[0]):
        for toks in blocks:
            rows.append(x[f, toks, :].sum(axis=0) / len(toks))
    return np.stack(rows) if rows else np.zeros((0, x.shape[-1]))


def block_scores(q_pooled: np.ndarray, k_pooled: np.ndarray) -> np.ndarray:
    """s[b, j] = q_pooled[b] . k_pooled[j] / sqrt(D)."""
    d = q_pooled.shape[-1]
    return (q_pooled @ k_pooled.T) / math.sqrt(d)


def select_topk(scores_row: np.ndarray, k: int) -> np.ndarray:
    """The k best blocks by (score descending, block id ascending), returned in
    ascending block id."""
    order = sorted(range(len(scores_row)), key=lambda j: (-float(scores_row[j]), j))
    return np.asarray(sorted(order[:k]), dtype=np.int64)


def select_blocks(q: np.ndarray, k_win: np.ndarray, frame_h: int, frame_w: int,
                  ratio: float, use_sparse: bool = True, bh: int = 8, bw: int = 8, bt: int = 1):
    """Top-k local blocks for every query block.

    q:     [B, Fq * T_f, H, D] query chunk.
    k_win: [B, Fw * T_f, H, D] local window, frames oldest first (logical order).
    Fq and Fw are multiples of bt; block id = frame group * NB + block in group.
    Returns idx [B, H, QB, k] (ascending ids), scores [B, H, QB, N_L].
    """
    blocks = frame_blocks(frame_h, frame_w, bh, bw, bt)
    tf = bt * frame_h * frame_w      # tokens of one frame group
    B, nq, H, D = q.shape
    fq, fw = nq // tf, k_win.shape[1] // tf
    n_local = fw * len(blocks)
    k = topk_count(ratio, n_local, use_sparse)
    qb = fq * len(blocks)
    idx = np.zeros((B, H, qb, k), dtype=np.int64)
    scores = np.zeros((B, H, qb, n_local))
    for b in range(B):
        for h in range(H):
            qbar = pool_blocks(np.asarray(q[b, :, h, :], np.float64).reshape(fq, tf, D), blocks)
            kbar = pool_blocks(np.asarray(k_win[b, :, h, :], np.float64).reshape(fw, tf, D), blocks)
            s = block_scores(qbar, kbar)
            scores[b, h] = s
            for i in range(qb):
                idx[b, h, i] = select_topk(s[i], k)
    return idx, scores


# ---------------------------------------------------------------------------------------
# Attention (pith abstract: PBSA attends to the persistent blocks and the selected local
# neighbourhood; project page call attn(query, key_persistent, value_persistent,
# key_local, value_local))
# ---------------------------------------------------------------------------------------
def attend_rows(q_rows: np.ndarray, keys: np.ndarray, values: np.ndarray):
    """Softmax attention of some query rows over a key set, scale 1/sqrt(D).

    Returns (O [n, D], lse [n] natural log, P [n, m] probabilities)."""
    d = q_rows.shape[-1]
    z = (q_rows @ keys.T) / math.sqrt(d)
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    denom = e.sum(axis=1, keepdims=True)
    p = e / denom
    return p @ values, (zmax + np.log(denom))[:, 0], p


def _persistent_keys(k_pers, v_pers, pers_len, b, h):
    """Valid rows of the occupied slots, slot order, with the owning slot of each row."""
    ks, vs, owner = [], [], []
    for s in range(pers_len.shape[2]):
        n = int(pers_len[b, h, s])
        if n > 0:
            ks.append(np.asarray(k_pers[b, h, s, :n], np.float64))
            vs.append(np.asarray(v_pers[b, h, s, :n], np.float64))
            owner.append(np.full(n, s))
    D = k_pers.shape[-1]
    if not ks:
        return np.zeros((0, D)), np.zeros((0, D)), np.zeros(0, dtype=np.int64)
    return np.concatenate(ks), np.concatenate(vs), np.concatenate(owner)


def _local_keys(k_win, v_win, b, h, ids, blocks, tf):
    """Tokens of the selected local blocks (logical ids), with the owning block of each."""
    nbf = len(blocks)
    ks, vs, owner = [], [], []
    for j in ids:
        f, i = divmod(int(j), nbf)
        toks = f * tf + blocks[i]
        ks.append(np.asarray(k_win[b, toks, h, :], np.float64))
        vs.append(np.asarray(v_win[b, toks, h, :], np.float64))
        owner.append(np.full(len(toks), int(j)))
    D = k_win.shape[-1]
    if not ks:
        return np.zeros((0, D)), np.zeros((0, D)), np.zeros(0, dtype=np.int64)
    return np.concatenate(ks), np.concatenate(vs), np.concatenate(owner)


def attn_fwd(q, k_pers, v_pers, pers_len, k_win, v_win, idx, frame_h, frame_w,
             bh=8, bw=8, heads=None, qblocks=None, bt=1):
    """PBSA forward.

    q [B, Nq, H, D]; k_pers/v_pers [B, H, S, 64, D] with pers_len [B, H, S];
    k_win/v_win [B, N_L_tokens, H, D] (logical window order); idx [B, H, QB, k].

    Every query token of query block b attends to all valid rows of all occupied
    persistent slots and to the valid tokens of the local blocks idx[b].
    Returns O [B, Nq, H, D], lse [B, H, Nq], mass_pers [B, H, S], mass_local [B, H, N_L]
    where mass is the probability summed over the query rows of this chunk, per block.
    `heads` (list of (b, h)) and `qblocks` (list of query block ids) restrict the work to
    a sample; rows outside it are left NaN in O and lse.  Blocks are bt x bh x bw.
    """
    blocks = frame_blocks(frame_h, frame_w, bh, bw, bt)
    tf = bt * frame_h * frame_w      # tokens of one frame group
    nbf = len(blocks)
    B, nq, H, D = q.shape
    S = pers_len.shape[2]
    n_local = (k_win.shape[1] // tf) * nbf
    O = np.full((B, nq, H, D), np.nan)
    lse = np.full((B, H, nq), np.nan)
    mass_pers = np.zeros((B, H, S))
    mass_local = np.zeros((B, H, n_local))
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        kp, vp, own_p = _persistent_keys(k_pers, v_pers, pers_len, b, h)
        qbs = range(idx.shape[2]) if qblocks is None else qblocks
        for qbi in qbs:
            f, i = divmod(qbi, nbf)
            toks = f * tf + blocks[i]
            kl, vl, own_l = _local_keys(k_win, v_win, b, h, idx[b, h, qbi], blocks, tf)
            keys = np.concatenate([kp, kl])
            vals = np.concatenate([vp, vl])
            o, l, p = attend_rows(np.asarray(q[b, toks, h, :], np.float64), keys, vals)
            O[b, toks, h, :] = o
            lse[b, h, toks] = l
            colsum = p.sum(axis=0)
            np.add.at(mass_pers[b, h], own_p, colsum[:len(kp)])
            np.add.at(mass_local[b, h], own_l, colsum[len(kp):])
    return O, lse, mass_pers, mass_local


# ---------------------------------------------------------------------------------------
# Memory update (pith abstract: persistent blocks are compressed, preserved and updated;
# algorithm fragment: the t=0 pass updates P and L)
# ---------------------------------------------------------------------------------------
def cache_update(k_pers, v_pers, pers_len, pers_score, pers_src, k_win, v_win, mass_local,
                 n_evict_frames, first_frame_global, frame_h, frame_w, bh=8, bw=8, bt=1,
                 n_sink=0):
    """Slide the window by n_evict_frames and merge the evicted blocks into the
    persistent set by accumulated attention mass.

    Inputs (numpy copies are made; nothing is modified in place):
      k_pers, v_pers [B, H, S, 64, D]; pers_len, pers_src [B, H, S] int; pers_score
      [B, H, S] float (accumulated mass of each slot); k_win, v_win [B, N, H, D] in
      logical window order; mass_local [B, H, N_L] by logical block id;
      first_frame_global: global frame number of the oldest window frame.

    Rule (reading):
      candidates = occupied slots in slot order, then the evicted blocks (logical ids
      0 .. n_evict_frames*NB_f - 1) in id order; order them by score descending, ties by
      candidate position; keep the first min(S, #candidates).  Kept slots stay where they
      are.  Free slots are the slots empty before the update in ascending order, then
      the dropped slots in ascending order.  Kept evicted blocks, in id order, fill the
      free slots in that order: the slot receives the block's tokens (raster order inside
      the block), its length, its mass as score and its global id
      (global frame group * NB + block in group, the group of global frames
      bt*g .. bt*g + bt - 1 being number g) as source.  Dropped slots not refilled end
      empty (length 0, score 0, source -1).  n_evict_frames and first_frame_global are
      multiples of bt.  The first n_sink slots hold sink blocks (sink_slots): they are
      neither candidates nor free slots, and S counts only the slots after them.

    Returns dict(k_pers, v_pers, pers_len, pers_score, pers_src, updates) where updates
    [b][h] is the list of (slot, logical block id) admissions in admission order.
    """
    blocks = frame_blocks(frame_h, frame_w, bh, bw, bt)
    nbf = len(blocks)
    tf = bt * frame_h * frame_w      # tokens of one frame group
    if n_evict_frames % bt or first_frame_global % bt:
        raise ValueError("frame counts must be multiples of the block's frame count")
    kp = np.array(k_pers, dtype=np.float64)
    vp = np.array(v_pers, dtype=np.float64)
    plen = np.array(pers_len, dtype=np.int64)
    pscore = np.array(pers_score, dtype=np.float64)
    psrc = np.array(pers_src, dtype=np.int64)
    B, H, S_all = plen.shape
    S = S_all - n_sink                  # slots that take part in the merge
    n_ev = n_evict_frames // bt * nbf
    updates = [[None] * H for _ in range(B)]
    for b in range(B):
        for h in range(H):
            mergeable = range(n_sink, S_all)
            occupied = [s for s in mergeable if plen[b, h, s] > 0]
            cands = [("slot", s, float(pscore[b, h, s])) for s in occupied]
            cands += [("block", j, float(mass_local[b, h, j])) for j in range(n_ev)]
            order = sorted(range(len(cands)), key=lambda c: (-cands[c][2], c))
            kept = set(order[:min(S, len(cands))])
            dropped = [cands[c][1] for c in range(len(occupied)) if c not in kept]
            free = [s for s in mergeable if plen[b, h, s] == 0] + sorted(dropped)
            for s in dropped:
                plen[b, h, s] = 0
                pscore[b, h, s] = 0.0
                psrc[b, h, s] = -1
                kp[b, h, s] = 0.0
                vp[b, h, s] = 0.0
            admitted = [cands[c][1] for c in range(len(occupied), len(cands)) if c in kept]
            ups = []
            for j, s in zip(admitted, free):
                f, i = divmod(j, nbf)
                toks = f * tf + blocks[i]
                n = len(toks)
                kp[b, h, s] = 0.0
                vp[b, h, s] = 0.0
                kp[b, h, s, :n] = np.asarray(k_win[b, toks, h, :], np.float64)
                vp[b, h, s, :n] = np.asarray(v_win[b, toks, h, :], np.float64)
                plen[b, h, s] = n
                pscore[b, h, s] = float(mass_local[b, h, j])
                psrc[b, h, s] = (first_frame_global // bt + f) * nbf + i
                ups.append((s, j))
            updates[b][h] = ups
    return dict(k_pers=kp, v_pers=vp, pers_len=plen, pers_score=pscore, pers_src=psrc,
                updates=updates)


# ---------------------------------------------------------------------------------------
# Backward (project page: full gradient support for training).  The selection is held
# fixed; gradients flow through the attention only.
# ---------------------------------------------------------------------------------------
def attn_bwd(q, k_pers, v_pers, pers_len, k_win, v_win, idx, dO, frame_h, frame_w,
             bh=8, bw=8, qblocks=None, bt=1):
    """Gradients of L = sum(O * dO) for the PBSA forward with the selection idx fixed.

    For each query block: P = softmax(q k^T / sqrt(D)) over its key set,
    dV += P^T dO, dP = dO V^T, dS = P * (dP - rowsum(P * dP)),
    dQ = dS K / sqrt(D), dK += dS^T Q / sqrt(D).
    Returns dQ [B, Nq, H, D], dK_pers/dV_pers [B, H, S, 64, D] (zero past each slot's
    length), dK_win/dV_win [B, N_L_tokens, H, D].  `qblocks` restricts the work to the
    contributions of those query blocks (a sample; the other rows of dQ stay zero).
    """
    blocks = frame_blocks(frame_h, frame_w, bh, bw, bt)
    tf = bt * frame_h * frame_w      # tokens of one frame group
    nbf = len(blocks)
    B, nq, H, D = q.shape
    S = pers_len.shape[2]
    sc = 1.0 / math.sqrt(D)
    dQ = np.zeros((B, nq, H, D))
    dKp = np.zeros(k_pers.shape)
    dVp = np.zeros(v_pers.shape)
    dKw = np.zeros(k_win.shape)
    dVw = np.zeros(v_win.shape)
    for b in range(B):
        for h in range(H):
            kp, vp, _ = _persistent_keys(k_pers, v_pers, pers_len, b, h)
            # destination (slot, row) of every persistent key row, in key order
            ps = np.concatenate([np.full(int(pers_len[b, h, s]), s) for s in range(S)]
                                + [np.zeros(0, dtype=np.int64)]).astype(np.int64)
            pr = np.concatenate([np.arange(int(pers_len[b, h, s])) for s in range(S)]
                                + [np.zeros(0, dtype=np.int64)]).astype(np.int64)
            for qbi in (range(idx.shape[2]) if qblocks is None else qblocks):
                f, i = divmod(qbi, nbf)
                toks = f * tf + blocks[i]
                ids = idx[b, h, qbi]
                kl, vl, _ = _local_keys(k_win, v_win, b, h, ids, blocks, tf)
                ltok = np.concatenate([(int(j) // nbf) * tf + blocks[int(j) % nbf] for j in ids]) \
                    if len(ids) else np.zeros(0, dtype=np.int64)
                keys = np.concatenate([kp, kl])
                vals = np.concatenate([vp, vl])
                qr = np.asarray(q[b, toks, h, :], np.float64)
                gr = np.asarray(dO[b, toks, h, :], np.float64)
                _, _, p = attend_rows(qr, keys, vals)
                dv = p.T @ gr
                dp = gr @ vals.T
                ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
                dQ[b, toks, h, :] += ds @ keys * sc
                dk = ds.T @ qr * sc
                npers = len(kp)
                np.add.at(dKp[b, h], (ps, pr), dk[:npers])
                np.add.at(dVp[b, h], (ps, pr), dv[:npers])
                np.add.at(dKw[b, :, h, :], ltok, dk[npers:])
                np.add.at(dVw[b, :, h, :], ltok, dv[npers:])
    return dQ, dKp, dVp, dKw, dVw


# ---------------------------------------------------------------------------------------
# The t=0 KV pass of one chunk, end to end (pith.science page, algorithm fragment in the
# reference list: the cache pass "applies PBSA with top-k and updates P and L"; abstract:
# the persistent blocks are preserved and updated as the window slides)
# ---------------------------------------------------------------------------------------
def evict_count(frames_in_window: int, chunk_frames: int, window_frames: int) -> int:
    """Frames that leave the window after a chunk's pass so that the next chunk fits.

    Reading: the window holds window_frames frames including the current chunk; after the
    pass, if frames_in_window + chunk_frames > window_frames, the oldest
    frames_in_window + chunk_frames - window_frames frames are evicted (for a 6-frame
    window and 3-frame chunks: nothing after chunk 0, then 3 frames after every chunk)."""
    return max(0, frames_in_window + chunk_frames - window_frames)


def append_frames(state, k_new, v_new, sink_frames, frame_h, frame_w, bh=8, bw=8, bt=1):
    """New frames join the cache (algorithm fragment: each chunk's frames enter the KV
    cache).  The first frame appended has global number first_frame_global + the window's
    frame count.  Frames whose global number is below sink_frames are sink frames
    (sink_slots): each of their blocks is written, whole, into its reserved slot
    (slot = global frame group * NB + block in group), with its token count as length,
    score 0 and its global id as source, and they do not enter the window; sink frames
    come first in a sequence, so the window is still empty then and its oldest frame
    becomes the first frame after them.  Every other frame joins the window after its
    newest frame.  Returns the new state; the input is not modified."""
    blocks = frame_blocks(frame_h, frame_w, bh, bw, bt)
    nbf = len(blocks)
    tf = frame_h * frame_w
    k_new = np.asarray(k_new, np.float64)
    v_new = np.asarray(v_new, np.float64)
    n = k_new.shape[1] // tf
    win_frames = state.win_k.shape[1] // tf
    g0 = state.first_frame_global + win_frames
    if g0 % bt or n % bt:
        raise ValueError("frames are appended in whole frame groups")
    n_sink_new = max(0, min(n, sink_frames - g0))
    if n_sink_new and win_frames:
        raise ValueError("sink frames come before every window frame")
    kp, vp = state.k_pers.copy(), state.v_pers.copy()
    plen, pscore, psrc = state.pers_len.copy(), state.pers_score.copy(), state.pers_src.copy()
    B, H = plen.shape[:2]
    for f in range(0, n_sink_new, bt):                       # one frame group at a time
        grp = (g0 + f) // bt
        for i, toks in enumerate(blocks):
            s = grp * nbf + i
            kp[:, :, s] = 0.0
            vp[:, :, s] = 0.0
            for b in range(B):
                for h in range(H):
                    kp[b, h, s, :len(toks)] = k_new[b, f * tf + toks, h, :]
                    vp[b, h, s, :len(toks)] = v_new[b, f * tf + toks, h, :]
            plen[:, :, s] = len(toks)
            pscore[:, :, s] = 0.0
            psrc[:, :, s] = s
    rest = slice(n_sink_new * tf, n * tf)
    return DecodeState(np.concatenate([state.win_k, k_new[:, rest]], 1),
                       np.concatenate([state.win_v, v_new[:, rest]], 1),
                       np.concatenate([state.win_mass, np.zeros((B, H, (n - n_sink_new) // bt * nbf))], 2),
                       kp, vp, plen, pscore, psrc, state.first_frame_global + n_sink_new)


class DecodeState:
    """Cache state between chunks, in the oracle's own plain layout (one batch item list
    entry per array axis as in the other oracle functions):

      win_k, win_v   [B, frames * T_f, H, D] window tokens, oldest frame first
      win_mass       [B, H, frames * NB_f]   accumulated mass of every window block
      k_pers, v_pers [B, H, S, 64, D]; pers_len, pers_src [B, H, S]; pers_score [B, H, S]
      first_frame_global: global frame number of the oldest window frame
    """

    def __init__(self, win_k, win_v, win_mass, k_pers, v_pers, pers_len, pers_score, pers_src,
                 first_frame_global=0):
        self.win_k = np.asarray(win_k, np.float64)
        self.win_v = np.asarray(win_v, np.float64)
        self.win_mass = np.asarray(win_mass, np.float64)
        self.k_pers = np.asarray(k_pers, np.float64)
        self.v_pers = np.asarray(v_pers, np.float64)
        self.pers_len = np.asarray(pers_len, np.int64)
        self.pers_score = np.asarray(pers_score, np.float64)
        self.pers_src = np.asarray(pers_src, np.int64)
        self.first_frame_global = int(first_frame_global)

    @classmethod
    def empty(cls, B, H, D, S, frame_h, frame_w, bh=8, bw=8):
        """A rollout's start: empty window, empty persistent cache (64-row slots)."""
        return cls(np.zeros((B, 0, H, D)), np.zeros((B, 0, H, D)), np.zeros((B, H, 0)),
                   np.zeros((B, H, S, 64, D)), np.zeros((B, H, S, 64, D)),
                   np.zeros((B, H, S), np.int64), np.zeros((B, H, S)),
                   np.full((B, H, S), -1, np.int64))


def decode_step(state: DecodeState, q, k_chunk, v_chunk, ratio, window_frames, frame_h,
                frame_w, use_sparse=True, idx=None, bh=8, bw=8, bt=1, sink_frames=0):
    """One chunk's cache pass, in the order of the algorithm fragment:

      1. the chunk's frames join the cache (append_frames; reading: before its attention,
         so the window includes the current chunk; sink frames go to their slots);
      2. top-k block selection over the window (select_blocks), unless `idx` is given
         (a caller may pass another implementation's selection to compare the rest of the
         step on equal terms);
      3. the PBSA forward with block mass (attn_fwd);
      4. the masses are accumulated: every window block and every persistent slot adds the
         probability mass it received in this pass (reading: per head, never decayed);
      5. slide: evict_count(frames, chunk frames, window_frames) oldest frames leave the
         window, and their blocks are merged into the persistent cache by accumulated mass
         (cache_update, the sink slots taking no part); the evicted blocks' masses leave
         with them.

    Returns (new_state, out) with out = dict(idx, scores, O, lse, mass_pers, mass_local,
    n_evict, updates).  The input state is not modified.
    """
    nbf = len(frame_blocks(frame_h, frame_w, bh, bw, bt))
    tf = frame_h * frame_w
    chunk_frames = np.asarray(k_chunk).shape[1] // tf
    n_sink = sink_slots(sink_frames, frame_h, frame_w, bh, bw, bt)
    appended = append_frames(state, k_chunk, v_chunk, sink_frames, frame_h, frame_w, bh, bw, bt)
    frames = appended.win_k.shape[1] // tf
    if frames > window_frames:
        raise ValueError("the window has no room for the chunk")
    win_k, win_v, win_mass = appended.win_k, appended.win_v, appended.win_mass
    B, H = state.pers_len.shape[:2]
    scores = None
    if idx is None:
        idx, scores = select_blocks(q, win_k, frame_h, frame_w, ratio, use_sparse, bh, bw, bt)
    O, lse, mass_pers, mass_local = attn_fwd(q, appended.k_pers, appended.v_pers,
                                             appended.pers_len, win_k, win_v, idx, frame_h,
                                             frame_w, bh, bw, bt=bt)
    win_mass = win_mass + mass_local
    pers_score = appended.pers_score + mass_pers
    n_ev = evict_count(frames, chunk_frames, window_frames)
    out = dict(idx=idx, scores=scores, O=O, lse=lse, mass_pers=mass_pers,
               mass_local=mass_local, n_evict=n_ev, updates=[[[] for _ in range(H)] for _ in range(B)],
               pers_score_before_merge=pers_score, win_mass_before_merge=win_mass)
    if n_ev == 0:
        new = DecodeState(win_k, win_v, win_mass, appended.k_pers, appended.v_pers,
                          appended.pers_len, pers_score, appended.pers_src,
                          appended.first_frame_global)
        return new, out
    r = cache_update(appended.k_pers, appended.v_pers, appended.pers_len, pers_score,
                     appended.pers_src, win_k, win_v, win_mass, n_ev,
                     appended.first_frame_global, frame_h, frame_w, bh, bw, bt, n_sink)
    out["updates"] = r["updates"]
    new = DecodeState(win_k[:, n_ev * tf:], win_v[:, n_ev * tf:], win_mass[:, :, n_ev // bt * nbf:],
                      r["k_pers"], r["v_pers"], r["pers_len"], r["pers_score"], r["pers_src"],
                      appended.first_frame_global + n_ev)
    return new, out
