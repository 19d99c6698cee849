"""Seeded synthetic inputs for PBSA tests and benchmarks.

The shapes follow the Sparse Forcing project page (boxunxu.top/SparseForcing), usage
snippet of ``SparseForcingAttention``: cache sizes in tokens (total 18720, local 9360,
persistent 9360), ``sparse_kv_block_size=[1, 8, 8]``, ``max_seq_len=32760`` and
``local_block_sparse_topk_ratio=0.125``.  The values are random normals.

This module only draws numbers and lays them out in the storage formats of the C ABI
(``include/pbsa.h``).  It computes nothing of the attention method: no pooling, scoring,
selection, softmax, mass or merge.  Both the CUDA path and the CPU oracle receive the
tensors it returns; neither imports the other.
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "block_extents", "decode_inputs", "rollout_chunk",
           "rollout_chunk_hot", "training_inputs", "slot_count"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: the page's constructor arguments plus the frame grid."""

    name: str
    B: int
    H: int
    D: int
    frame_h: int
    frame_w: int
    local_cache_size: int       # tokens in the sliding local window
    persistent_cache_size: int  # tokens of persistent blocks
    total_cache_size: int       # local + persistent
    max_seq_len: int
    q_frames: int               # frames per query chunk
    topk_ratio: float           # local_block_sparse_topk_ratio
    use_sparse: bool = True     # use_local_block_sparse_attn
    block: tuple = (1, 8, 8)    # sparse_kv_block_size [t, h, w]
    value_std: float = 1.0      # std of every Q/K/V entry
    bias_fraction: float = 0.0  # fraction of key blocks given a shared bias direction
    bias_sigma: float = 2.0     # bias length, in units of value_std
    seed: int = 0
    chunks: int = 1             # chunks in a rollout or training sequence

    @property
    def tokens_per_frame(self) -> int:
        return self.frame_h * self.frame_w

    @property
    def window_frames(self) -> int:
        return self.local_cache_size // self.tokens_per_frame

    @property
    def nq(self) -> int:
        return self.q_frames * self.tokens_per_frame


WORKLOADS = {
    # Tiny correctness case: 16x16 grid (four 8x8 blocks per frame), 4-frame window,
    # 8 persistent blocks, 1-frame chunk, ratio 0.25, entries 0.5*N(0,1).
    "tiny": Workload("tiny", B=1, H=2, D=64, frame_h=16, frame_w=16,
                     local_cache_size=1024, persistent_cache_size=512,
                     total_cache_size=1536, max_seq_len=4096, q_frames=1,
                     topk_ratio=0.25, value_std=0.5, seed=0),
    # Page-sized decode step: 30x52 grid (1560 tokens/frame), 6-frame window,
    # 9360 persistent tokens, 3-frame chunk, ratio 0.125, 5% biased key blocks.
    "decode": Workload("decode", B=1, H=12, D=128, frame_h=30, frame_w=52,
                       local_cache_size=9360, persistent_cache_size=9360,
                       total_cache_size=18720, max_seq_len=32760, q_frames=3,
                       topk_ratio=0.125, bias_fraction=0.05, seed=1),
    # The page-sized decode step with the project page's [3,4,4] blocks (3 frames x 4 x 4
    # tokens): 104 blocks per 3-frame group, 208 slots, 208 window blocks, k = 26.
    "decode344": Workload("decode344", B=1, H=12, D=128, frame_h=30, frame_w=52,
                          local_cache_size=9360, persistent_cache_size=9360,
                          total_cache_size=18720, max_seq_len=32760, q_frames=3,
                          topk_ratio=0.125, block=(3, 4, 4), bias_fraction=0.05, seed=4),
    # Rollout: decode shapes, 20 chunks, empty persistent cache at the start.
    "rollout": Workload("rollout", B=1, H=12, D=128, frame_h=30, frame_w=52,
                        local_cache_size=9360, persistent_cache_size=9360,
                        total_cache_size=18720, max_seq_len=32760, q_frames=3,
                        topk_ratio=0.125, seed=2, chunks=20),
    # Training: 21 frames = 32760 tokens in 7 chunks of 3 frames.
    "train": Workload("train", B=1, H=12, D=128, frame_h=30, frame_w=52,
                      local_cache_size=9360, persistent_cache_size=9360,
                      total_cache_size=18720, max_seq_len=32760, q_frames=3,
                      topk_ratio=0.125, seed=3, chunks=7),
}


def block_extents(frame_h: int, frame_w: int, bh: int = 8, bw: int = 8):
    """(rows, cols) of every block of one frame, in block order (row of blocks, then column).

    Edge blocks are clipped to the frame, so a 30x52 frame has 8x8, 8x4, 6x8 and 6x4
    blocks.  A block of bt frames has bt * rows * cols tokens.  Used only to lay out the
    synthetic persistent store and the biased blocks.
    """
    out = []
    for y0 in range(0, frame_h, bh):
        for x0 in range(0, frame_w, bw):
            out.append((min(bh, frame_h - y0), min(bw, frame_w - x0)))
    return out


def slot_count(wl: Workload) -> int:
    """Number of 64-row persistent slots for the workload's persistent_cache_size."""
    bt = wl.block[0]
    tg = wl.tokens_per_frame * bt
    nbf = len(block_extents(wl.frame_h, wl.frame_w, wl.block[1], wl.block[2]))
    if wl.persistent_cache_size % tg == 0:
        return wl.persistent_cache_size // tg * nbf
    cap = bt * wl.block[1] * wl.block[2]
    return -(-wl.persistent_cache_size // cap)


def _normal(gen, shape, std):
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std


def _unit(gen, d):
    u = torch.randn(d, generator=gen, dtype=torch.float64)
    return (u / u.norm()).to(torch.float32)


def _bias_local(gen, x, wl, frames):
    """Add bias_sigma*value_std*u to every token of a seeded subset of key blocks.

    x is [B, frames*T_f, H, D]; the subset has round(bias_fraction * blocks) blocks per
    (batch, head) and u is one unit vector per (batch, head).
    """
    if wl.bias_fraction <= 0:
        return
    bt, bh, bw = wl.block
    ext = block_extents(wl.frame_h, wl.frame_w, bh, bw)
    nbx = -(-wl.frame_w // bw)
    nblk = frames // bt * len(ext)
    nb = int(round(wl.bias_fraction * nblk))
    xv = x.view(wl.B, frames, wl.frame_h, wl.frame_w, wl.H, wl.D)
    for b in range(wl.B):
        for h in range(wl.H):
            u = _unit(gen, wl.D) * (wl.bias_sigma * wl.value_std)
            pick = torch.randperm(nblk, generator=gen)[:nb].tolist()
            for j in pick:
                f, i = divmod(j, len(ext))
                by, bx = divmod(i, nbx)
                xv[b, f * bt:f * bt + bt, by * bh:by * bh + bh, bx * bw:bx * bw + bw, h, :] += u


def _persistent(gen, wl, n_slots, filled_slots):
    """Persistent store [B,H,S,64,D] whose first filled_slots slots hold blocks with the
    frame's block-size pattern; rows past each slot's length are zero."""
    ext = block_extents(wl.frame_h, wl.frame_w, wl.block[1], wl.block[2])
    k = torch.zeros(wl.B, wl.H, n_slots, 64, wl.D)
    v = torch.zeros(wl.B, wl.H, n_slots, 64, wl.D)
    length = torch.zeros(wl.B, wl.H, n_slots, dtype=torch.int32)
    for s in range(filled_slots):
        r, c = ext[s % len(ext)]
        length[:, :, s] = wl.block[0] * r * c
    for b in range(wl.B):
        for h in range(wl.H):
            for s in range(filled_slots):
                n = int(length[b, h, s])
                k[b, h, s, :n] = _normal(gen, (n, wl.D), wl.value_std)
                v[b, h, s, :n] = _normal(gen, (n, wl.D), wl.value_std)
    if wl.bias_fraction > 0:
        nb = int(round(wl.bias_fraction * filled_slots))
        for b in range(wl.B):
            for h in range(wl.H):
                u = _unit(gen, wl.D) * (wl.bias_sigma * wl.value_std)
                for s in torch.randperm(filled_slots, generator=gen)[:nb].tolist():
                    n = int(length[b, h, s])
                    k[b, h, s, :n] += u
    return k, v, length


def decode_inputs(wl: Workload, seed: int | None = None, persistent_filled: bool = True):
    """One decode step with a full window and (optionally) a full persistent cache.

    Returns a dict of CPU tensors:
      q        [B, q_frames*T_f, H, D] bf16
      k_local  [B, W*T_f, H, D] bf16, v_local likewise (ring with head 0, W frames held)
      k_pers   [B, H, S, 64, D] bf16, v_pers likewise; rows >= pers_len are zero
      pers_len [B, H, S] int32
    """
    gen = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    tf = wl.tokens_per_frame
    W = wl.window_frames
    q = _normal(gen, (wl.B, wl.q_frames * tf, wl.H, wl.D), wl.value_std)
    kl = _normal(gen, (wl.B, W * tf, wl.H, wl.D), wl.value_std)
    vl = _normal(gen, (wl.B, W * tf, wl.H, wl.D), wl.value_std)
    _bias_local(gen, kl, wl, W)
    S = slot_count(wl)
    kp, vp, plen = _persistent(gen, wl, S, S if persistent_filled else 0)
    bf = torch.bfloat16
    return dict(q=q.to(bf), k_local=kl.to(bf), v_local=vl.to(bf), k_pers=kp.to(bf),
                v_pers=vp.to(bf), pers_len=plen)


def rollout_chunk(wl: Workload, step: int):
    """Fresh Q, K, V for chunk `step` of a rollout: each [B, q_frames*T_f, H, D] bf16."""
    gen = torch.Generator().manual_seed(wl.seed * 1000003 + step)
    shape = (wl.B, wl.q_frames * wl.tokens_per_frame, wl.H, wl.D)
    bf = torch.bfloat16
    q = _normal(gen, shape, wl.value_std).to(bf)
    k = _normal(gen, shape, wl.value_std).to(bf)
    v = _normal(gen, shape, wl.value_std).to(bf)
    return q, k, v


def rollout_chunk_hot(wl: Workload, step: int, q_bias: float = 4.0, hot_bias: float = 4.0,
                      hot_fraction: float = 0.1):
    """Like rollout_chunk, but every query token carries q_bias * u and a seeded
    hot_fraction of the chunk's key blocks carry hot_bias * u on every token, u being one
    seeded unit vector per (batch, head) shared by all chunks: a stream in which some new
    blocks keep drawing most of the queries' attention."""
    q, k, v = rollout_chunk(wl, step)
    gu = torch.Generator().manual_seed(wl.seed * 7919 + 1)
    u = torch.stack([torch.stack([_unit(gu, wl.D) for _ in range(wl.H)]) for _ in range(wl.B)])
    gen = torch.Generator().manual_seed(wl.seed * 1000033 + step)
    qf = q.float() + q_bias * u[:, None]
    kf = k.float()
    ext = block_extents(wl.frame_h, wl.frame_w, wl.block[1], wl.block[2])
    nbx = -(-wl.frame_w // wl.block[2])
    nblk = wl.q_frames * len(ext)
    nhot = max(1, int(round(hot_fraction * nblk)))
    kv = kf.view(wl.B, wl.q_frames, wl.frame_h, wl.frame_w, wl.H, wl.D)
    bh, bw = wl.block[1], wl.block[2]
    for b in range(wl.B):
        for h in range(wl.H):
            for j in torch.randperm(nblk, generator=gen)[:nhot].tolist():
                f, i = divmod(j, len(ext))
                by, bx = divmod(i, nbx)
                kv[b, f, by * bh:by * bh + bh, bx * bw:bx * bw + bw, h, :] += hot_bias * u[b, h]
    bf = torch.bfloat16
    return qf.to(bf), kf.to(bf), v


def training_inputs(wl: Workload, frames: int | None = None):
    """A training sequence: Q, K, V, dO over `frames` frames ([B, frames*T_f, H, D] bf16)
    and a full synthetic persistent store."""
    gen = torch.Generator().manual_seed(wl.seed)
    frames = wl.chunks * wl.q_frames if frames is None else frames
    shape = (wl.B, frames * wl.tokens_per_frame, wl.H, wl.D)
    bf = torch.bfloat16
    q = _normal(gen, shape, wl.value_std).to(bf)
    k = _normal(gen, shape, wl.value_std).to(bf)
    v = _normal(gen, shape, wl.value_std).to(bf)
    do = _normal(gen, shape, wl.value_std).to(bf)
    S = slot_count(wl)
    kp, vp, plen = _persistent(gen, wl, S, S)
    return dict(q=q, k=k, v=v, do=do, k_pers=kp.to(bf), v_pers=vp.to(bf), pers_len=plen)
