"""Stateful Python face of the PBSA C ABI, shaped like the project page's
``SparseForcingAttention`` (boxunxu.top/SparseForcing, usage snippet).

The object owns the device-resident caches (local ring, persistent slots, block masses)
and the workspaces; torch is used only to allocate them and to move the caller's tensors.
Every step of the method runs in the CUDA kernels behind ``pbsa.pbsa_*``.

Typical t=0 decode pass for one chunk (pith.science page, algorithm fragment: the KV pass
applies PBSA with top-k and updates P and L):

    attn.append(k_chunk, v_chunk)        # new frames enter the ring (the window), their key
                                         # means the key-mean cache; sink frames their slots
    out = attn(q_chunk, accumulate_mass=True)   # select + forward (+ block mass)
    attn.slide()                         # evict old frames, merge them into P
"""
from __future__ import annotations

import torch

from . import pbsa as P


class SparseForcingAttention:
    def __init__(self, B: int, H: int, D: int, frame_h: int, frame_w: int,
                 total_cache_size: int = 18720, local_cache_size: int = 9360,
                 persistent_cache_size: int = 9360, kv_cache_mode: str = "sparse_forcing",
                 sparse_kv_block_size=(1, 8, 8), max_seq_len: int = 32760,
                 use_local_block_sparse_attn: bool = True,
                 local_block_sparse_topk_ratio: float = 0.125, chunk_frames: int = 3,
                 sink_frames: int = 0, device="cuda"):
        # kv_cache_mode="dense": one window of total_cache_size tokens, no persistent slots
        # (S = 0), every block attended; slide() then only drops the oldest frames.
        # sink_frames: the first frames of the sequence are kept in sink slots, attended by
        # every query and never evicted.
        self.cfg = P.make_config(B, H, D, frame_h, frame_w, total_cache_size, local_cache_size,
                                 persistent_cache_size, max_seq_len,
                                 local_block_sparse_topk_ratio, use_local_block_sparse_attn,
                                 sparse_kv_block_size, kv_cache_mode, sink_frames)
        P.pbsa_validate_config(self.cfg)
        self.B, self.H, self.D = B, H, D
        self.tf = frame_h * frame_w
        self.bt = int(sparse_kv_block_size[0])      # frames per block (a frame group)
        self.nbf = P.pbsa_blocks_per_frame(self.cfg)  # blocks per frame group
        self.W = P.pbsa_window_frames(self.cfg)
        self.S = P.pbsa_num_slots(self.cfg)
        self.n_sink = P.pbsa_sink_slots(self.cfg)
        if chunk_frames % self.bt:
            raise ValueError("chunk_frames must be a multiple of the block's frame count")
        self.chunk_frames = chunk_frames
        self.kmax = P.pbsa_topk_count(self.cfg, self.W)
        self.device = torch.device(device)
        dev = self.device
        bf = dict(dtype=torch.bfloat16, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        i32 = dict(dtype=torch.int32, device=dev)
        # caches
        self.k_local = torch.zeros(B, self.W * self.tf, H, D, **bf)
        self.v_local = torch.zeros(B, self.W * self.tf, H, D, **bf)
        self.k_pers = torch.zeros(B, H, self.S, 64, D, **bf)
        self.v_pers = torch.zeros(B, H, self.S, 64, D, **bf)
        self.pers_len = torch.zeros(B, H, self.S, **i32)
        self.pers_score = torch.zeros(B, H, self.S, **f32)
        self.pers_src = torch.full((B, H, self.S), -1, **i32)
        self.mass_local = torch.zeros(B, H, self.W // self.bt * self.nbf, **f32)
        self.kbar = torch.zeros(B, H, self.W // self.bt * self.nbf, D, **f32)   # key means by ring slot
        self.ring_head = 0
        self.local_frames = 0
        self.first_frame_global = 0   # global number of the oldest window frame
        self.frames_seen = 0          # frames appended so far (sink frames included)
        # per-chunk buffers
        qf = chunk_frames
        qb = qf // self.bt * self.nbf
        self.idx = torch.zeros(B, H, qb, self.kmax, **i32)
        self.cnt = torch.zeros(B, H, qb, **i32)
        self.out = torch.empty(B, qf * self.tf, H, D, **bf)
        self.lse = torch.empty(B, H, qf * self.tf, **f32)
        self.upd = torch.zeros(B, H, self.W // self.bt * self.nbf, 2, **i32)
        self.n_upd = torch.zeros(B, H, **i32)
        self.status = torch.zeros(1, **i32)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.ws_select = torch.empty(P.pbsa_workspace_size(self.cfg, P.PBSA_OP_SELECT, qf), **u8)
        self.ws_fwd = torch.empty(max(1, P.pbsa_workspace_size(self.cfg, P.PBSA_OP_FWD, qf)), **u8)
        self.ws_bwd = torch.empty(max(1, P.pbsa_workspace_size(self.cfg, P.PBSA_OP_BWD, qf)), **u8)
        self._grads = None

    # ------------------------------------------------------------------ cache plumbing
    def ring_slot(self, p: int) -> int:
        """Ring slot of window frame p (0 = oldest)."""
        return (self.ring_head + p) % self.W

    def frame_view(self, p: int, which: str = "k"):
        """[B, T_f, H, D] view of window frame p in the ring (writable, zero-copy)."""
        s = self.ring_slot(p)
        t = self.k_local if which == "k" else self.v_local
        return t[:, s * self.tf:(s + 1) * self.tf]

    def append(self, k_chunk: torch.Tensor, v_chunk: torch.Tensor):
        """The chunk's frames join the cache (the window must have room: call slide() first
        when it is full): sink frames go to their slots, the others after the newest window
        frame, their key means into the key-mean cache, all in one kernel.  Accepts device
        tensors, or host (pinned) tensors that are first copied to the device, of shape
        [B, frames*T_f, H, D] bf16."""
        n = k_chunk.shape[1] // self.tf
        n_sink = max(0, min(n, self.cfg.sink_frames - self.frames_seen))
        if self.local_frames + n - n_sink > self.W:
            raise ValueError("window full: slide() before append()")
        if k_chunk.device != self.device:
            k_chunk = k_chunk.to(self.device, non_blocking=True)
            v_chunk = v_chunk.to(self.device, non_blocking=True)
        P.pbsa_append_frames(self.cfg, k_chunk.contiguous(), v_chunk.contiguous(), n,
                             self.frames_seen, self.k_local, self.v_local,
                             (self.ring_head + self.local_frames) % self.W, self.kbar,
                             self.k_pers, self.v_pers, self.pers_len, self.pers_score,
                             self.pers_src)
        self.frames_seen += n
        self.local_frames += n - n_sink
        self.first_frame_global = self.frames_seen - self.local_frames

    def pool_window(self):
        """Recomputes the key-mean cache for every window frame, for callers that wrote the
        ring directly instead of through append()."""
        if self.local_frames:
            P.pbsa_pool_keys(self.cfg, self.k_local, self.ring_head, self.local_frames, self.kbar)

    def load_persistent(self, k_pers, v_pers, pers_len, pers_score=None, pers_src=None):
        self.k_pers.copy_(k_pers)
        self.v_pers.copy_(v_pers)
        self.pers_len.copy_(pers_len)
        if pers_score is not None:
            self.pers_score.copy_(pers_score)
        if pers_src is not None:
            self.pers_src.copy_(pers_src)

    # ------------------------------------------------------------------ the method
    def select(self, q: torch.Tensor, q_frames: int | None = None):
        """Top-k local blocks for the chunk, scored against the key-mean cache."""
        qf = self.chunk_frames if q_frames is None else q_frames
        P.pbsa_select_blocks_pooled(self.cfg, q, qf, self.kbar, self.local_frames, self.ring_head,
                                    self.idx, self.kmax, self.cnt, None, self.ws_select)

    def attend(self, q: torch.Tensor, accumulate_mass: bool = False, q_frames: int | None = None):
        qf = self.chunk_frames if q_frames is None else q_frames
        P.pbsa_attn_fwd(self.cfg, q, qf, self.k_pers, self.v_pers, self.pers_len, self.k_local,
                        self.v_local, self.local_frames, self.ring_head, self.idx, self.kmax,
                        self.cnt, self.out, self.lse,
                        self.mass_local if accumulate_mass else None,
                        self.pers_score if accumulate_mass else None,
                        self.ws_fwd if accumulate_mass else None, self.status)
        return self.out

    def __call__(self, q: torch.Tensor, accumulate_mass: bool = False):
        """Block selection then the PBSA forward; returns the output buffer."""
        self.select(q)
        return self.attend(q, accumulate_mass)

    def backward_buffers(self):
        """The fp32 gradient outputs (dq, dk_pers, dv_pers, dk_local, dv_local), allocated
        on first use."""
        if self._grads is None:
            f32 = dict(dtype=torch.float32, device=self.device)
            self._grads = (torch.zeros(self.out.shape, **f32),
                           torch.zeros(self.k_pers.shape, **f32),
                           torch.zeros(self.v_pers.shape, **f32),
                           torch.zeros(self.k_local.shape, **f32),
                           torch.zeros(self.v_local.shape, **f32))
        return self._grads

    def backward(self, q: torch.Tensor, dout: torch.Tensor):
        """Gradients of sum(out * dout) for the last forward (same caches, same selection).
        Returns (dq, dk_pers, dv_pers, dk_local, dv_local), fp32, owned by this object."""
        dq, dkp, dvp, dkl, dvl = self.backward_buffers()
        P.pbsa_attn_bwd(self.cfg, q, self.chunk_frames, self.k_pers, self.v_pers, self.pers_len,
                        self.k_local, self.v_local, self.local_frames, self.ring_head, self.idx,
                        self.kmax, self.cnt, self.out, self.lse, dout, dq, dkp, dvp, dkl, dvl,
                        self.ws_bwd, self.status)
        return self._grads

    def slide(self, n_evict_frames: int | None = None):
        """Evicts the oldest frames so that the next chunk fits, merging their blocks into
        the persistent cache by accumulated mass.  Returns the number evicted."""
        if n_evict_frames is None:
            n_evict_frames = max(0, self.local_frames + self.chunk_frames - self.W)
        if n_evict_frames == 0:
            return 0
        P.pbsa_cache_update(self.cfg, self.k_local, self.v_local, self.local_frames,
                            self.ring_head, self.mass_local, n_evict_frames,
                            self.first_frame_global, self.k_pers, self.v_pers, self.pers_len,
                            self.pers_score, self.pers_src, self.upd, self.n_upd)
        self.ring_head = (self.ring_head + n_evict_frames) % self.W
        self.local_frames -= n_evict_frames
        self.first_frame_global += n_evict_frames
        return n_evict_frames
