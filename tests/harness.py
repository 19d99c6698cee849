"""Host-side helpers for the PBSA tests: configs from workloads, buffer allocation, ring
<-> window bookkeeping and the comparison rules (tolerances, top-k re-verification)."""
from __future__ import annotations

import math

import numpy as np
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import Workload, slot_count

# Tolerances of the GPU path against the fp64 oracle.
FWD_MAX_ABS = 2e-2      # bf16 output, max |error|
FWD_REL_L2 = 1e-2       # bf16 output, ||error|| / ||oracle||
GRAD_REL_L2 = 3e-2      # gradients, relative L2
LSE_ABS = 1e-3          # fp32 log-sum-exp: fp32 accumulation of <= ~2e4 terms
MASS_REL = 1e-3         # fp32 masses: fp32 sums of fp32 exponentials
MASS_ABS = 1e-3
TOPK_MARGIN = 1e-3      # below this score margin the GPU's set is re-verified


def config(wl: Workload, **over):
    kw = dict(B=wl.B, H=wl.H, D=wl.D, frame_h=wl.frame_h, frame_w=wl.frame_w,
              total_cache_size=wl.total_cache_size, local_cache_size=wl.local_cache_size,
              persistent_cache_size=wl.persistent_cache_size, max_seq_len=wl.max_seq_len,
              local_block_sparse_topk_ratio=wl.topk_ratio,
              use_local_block_sparse_attn=wl.use_sparse, sparse_kv_block_size=wl.block)
    kw.update(over)
    return P.make_config(**kw)


def ring_to_window(ring, ring_head, local_frames, W, tf):
    """Logical window [B, local_frames*T_f, H, D] (oldest frame first) from a ring."""
    frames = [(ring_head + p) % W for p in range(local_frames)]
    idx = torch.cat([torch.arange(f * tf, (f + 1) * tf) for f in frames])
    return ring[:, idx.to(ring.device)]


def window_to_ring(win, ring_head, W, tf, out=None):
    """Places a logical window back into a ring of W frame slots (other slots zero)."""
    B, n, H, D = win.shape
    lf = n // tf
    ring = torch.zeros(B, W * tf, H, D, dtype=win.dtype, device=win.device) if out is None else out
    for p in range(lf):
        f = (ring_head + p) % W
        ring[:, f * tf:(f + 1) * tf] = win[:, p * tf:(p + 1) * tf]
    return ring


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


class Buffers:
    """Device outputs and workspaces for one decode step."""

    def __init__(self, cfg, wl: Workload, q_frames: int, local_frames: int, dev, idx_stride=None):
        self.cfg = cfg
        tf = wl.tokens_per_frame
        nbf = P.pbsa_blocks_per_frame(cfg)
        W = P.pbsa_window_frames(cfg)
        S = P.pbsa_num_slots(cfg)
        assert S == slot_count(wl)
        bt = cfg.block_t
        self.nbf, self.W, self.S, self.tf, self.bt = nbf, W, S, tf, bt
        self.qb = q_frames // bt * nbf
        self.nl = local_frames // bt * nbf
        self.k = P.pbsa_topk_count(cfg, local_frames)
        self.idx_stride = self.k if idx_stride is None else idx_stride
        B, H, D = wl.B, wl.H, wl.D
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.idx = torch.full((B, H, self.qb, self.idx_stride), -7, **i32)
        self.cnt = torch.zeros((B, H, self.qb), **i32)
        self.scores = torch.zeros((B, H, self.qb, self.nl), **f32)
        self.ws_sel = torch.empty(P.pbsa_workspace_size(cfg, P.PBSA_OP_SELECT, q_frames),
                                  dtype=torch.uint8, device=dev)
        self.ws_fwd = torch.empty(max(1, P.pbsa_workspace_size(cfg, P.PBSA_OP_FWD, q_frames)),
                                  dtype=torch.uint8, device=dev)
        self.ws_bwd = torch.empty(max(1, P.pbsa_workspace_size(cfg, P.PBSA_OP_BWD, q_frames)),
                                  dtype=torch.uint8, device=dev)
        self.out = torch.full((B, q_frames * tf, H, D), float("nan"), dtype=torch.bfloat16, device=dev)
        self.lse = torch.full((B, H, q_frames * tf), float("nan"), **f32)
        self.mass_local = torch.zeros((B, H, W // bt * nbf), **f32)
        self.mass_pers = torch.zeros((B, H, S), **f32)
        self.status = torch.zeros(1, **i32)


def run_select(buf, q, q_frames, k_local, local_frames, ring_head, scores=True):
    P.pbsa_select_blocks(buf.cfg, q, q_frames, k_local, local_frames, ring_head, buf.idx,
                         buf.idx_stride, buf.cnt, buf.scores if scores else None, buf.ws_sel)


def run_fwd(buf, q, q_frames, k_pers, v_pers, pers_len, k_local, v_local, local_frames,
            ring_head, mass=True):
    P.pbsa_attn_fwd(buf.cfg, q, q_frames, k_pers, v_pers, pers_len, k_local, v_local,
                    local_frames, ring_head, buf.idx, buf.idx_stride, buf.cnt, buf.out, buf.lse,
                    buf.mass_local if mass else None, buf.mass_pers if mass else None,
                    buf.ws_fwd if mass else None, buf.status)


def check_topk(idx_gpu, cnt_gpu, scores_orc, k, margin=TOPK_MARGIN):
    """GPU top-k sets against the oracle's scores.

    Where the oracle's gap between the k-th and (k+1)-th score exceeds `margin`, the set
    must equal the oracle's exactly; elsewhere every chosen block must score at least every
    unchosen block minus `margin`.  Returns the fraction compared exactly."""
    idx_gpu = np.asarray(idx_gpu)
    cnt_gpu = np.asarray(cnt_gpu)
    B, H, QB, NL = scores_orc.shape
    exact = 0
    for b in range(B):
        for h in range(H):
            for i in range(QB):
                assert cnt_gpu[b, h, i] == k
                got = idx_gpu[b, h, i, :k]
                assert np.all(np.diff(got) > 0), "indices must be strictly ascending"
                assert got.min() >= 0 and got.max() < NL
                s = scores_orc[b, h, i]
                order = sorted(range(NL), key=lambda j: (-s[j], j))
                want = sorted(order[:k])
                gap = s[order[k - 1]] - s[order[k]] if k < NL else math.inf
                if gap > margin:
                    assert list(got) == want, (b, h, i, list(got), want, gap)
                    exact += 1
                else:
                    chosen = set(int(x) for x in got)
                    lo = min(s[j] for j in chosen)
                    hi = max((s[j] for j in range(NL) if j not in chosen), default=-math.inf)
                    assert lo >= hi - margin, (b, h, i, lo, hi)
    return exact / (B * H * QB)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


def assert_close_bf16(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want).max()
    rl2 = rel_l2(got, want)
    assert err <= FWD_MAX_ABS and rl2 <= FWD_REL_L2, f"{what}: max abs {err:.3e}, rel L2 {rl2:.3e}"
    return err, rl2
