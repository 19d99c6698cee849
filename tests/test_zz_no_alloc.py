"""The workspace-free block selection (pbsa_select_blocks_noalloc) against the regular
one (pbsa_select_blocks), both called through the C ABI.

pbsa_select_blocks_noalloc exists for callers that cannot allocate device memory where
they select blocks (an engine plugin with a fixed memory plan, a decode loop that must not
call cudaMalloc); it keeps its scratch in a static device buffer shared by all calls.
The test runs two different selections in a row so that the second call reuses the
buffer the first one filled, and must give the same results whether this file runs
alone in a fresh process or after the other tests.  This file is named so that pytest
collects it last."""
import dataclasses

import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import WORKLOADS, decode_inputs
from tests.harness import config

pytestmark = pytest.mark.gpu


def _selection(cfg, wl, q, kl, local_frames, ring_head, noalloc, dev):
    nbf = P.pbsa_blocks_per_frame(cfg)
    qb, nl = wl.q_frames * nbf, local_frames * nbf
    k = P.pbsa_topk_count(cfg, local_frames)
    idx = torch.full((wl.B, wl.H, qb, k), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((wl.B, wl.H, qb), dtype=torch.int32, device=dev)
    sc = torch.zeros((wl.B, wl.H, qb, nl), dtype=torch.float32, device=dev)
    if noalloc:
        P.pbsa_select_blocks_noalloc(cfg, q, wl.q_frames, kl, local_frames, ring_head, idx, k,
                                     cnt, sc)
    else:
        ws = torch.empty(P.pbsa_workspace_size(cfg, P.PBSA_OP_SELECT, wl.q_frames),
                         dtype=torch.uint8, device=dev)
        P.pbsa_select_blocks(cfg, q, wl.q_frames, kl, local_frames, ring_head, idx, k, cnt, sc, ws)
    torch.cuda.synchronize()
    return idx, cnt, sc


def test_noalloc_selection_matches_workspace_selection_twice(cuda_dev):
    wl = WORKLOADS["decode"]
    cfg = config(wl)
    assert P.pbsa_workspace_size(cfg, P.PBSA_OP_SELECT, wl.q_frames) <= 8 << 20
    # two different selections back to back: the full window, then a 4-frame window at
    # another ring position of other data (the second call overwrites the first's scratch)
    cases = [(decode_inputs(wl), 6, 0), (decode_inputs(wl, seed=99), 4, 5)]
    for inp, lf, rh in cases:
        q = inp["q"].to(cuda_dev)
        kl = inp["k_local"].to(cuda_dev)
        want = _selection(cfg, wl, q, kl, lf, rh, False, cuda_dev)
        got = _selection(cfg, wl, q, kl, lf, rh, True, cuda_dev)
        assert torch.equal(got[0], want[0])
        assert torch.equal(got[1], want[1])
        assert torch.allclose(got[2], want[2], rtol=0, atol=1e-5)


def test_noalloc_rejects_selections_larger_than_its_buffer(cuda_dev):
    # batch 8 of the decode shapes needs ~12 MB of pooled means: more than the 8 MiB buffer
    wl = dataclasses.replace(WORKLOADS["decode"], B=8)
    cfg = config(wl)
    assert P.pbsa_workspace_size(cfg, P.PBSA_OP_SELECT, wl.q_frames) > 8 << 20
    dev = cuda_dev
    t = torch.zeros(16, dtype=torch.bfloat16, device=dev)
    i = torch.zeros(16, dtype=torch.int32, device=dev)
    with pytest.raises(P.PBSAError) as e:
        P.pbsa_select_blocks_noalloc(cfg, t, wl.q_frames, t, 6, 0, i, 21, i, None)
    assert e.value.code == P.PBSA_ERR_UNSUPPORTED
    assert "8 MiB" in P.pbsa_last_error()
