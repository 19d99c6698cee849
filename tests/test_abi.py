"""The C-ABI library loads, exports every function include/pbsa.h declares, and its
host-only logic (validation, geometry, workspace sizes, argument checks) works without a
GPU.  No test here launches a kernel."""
import ctypes
import dataclasses

import pytest

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import WORKLOADS, slot_count
from oracle import pbsa_oracle as orc
from tests.harness import config


def test_library_exports_every_header_symbol():
    names = P.header_symbols()
    assert len(names) >= 12
    lib = ctypes.CDLL(P.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("name", ["tiny", "decode", "rollout", "train", "decode344"])
def test_geometry_matches_oracle(name):
    wl = WORKLOADS[name]
    cfg = config(wl)
    P.pbsa_validate_config(cfg)
    bt, bh, bw = wl.block
    nbf = len(orc.frame_blocks(wl.frame_h, wl.frame_w, bh, bw, bt))
    assert P.pbsa_blocks_per_frame(cfg) == nbf
    assert P.pbsa_window_frames(cfg) == wl.window_frames
    assert P.pbsa_num_slots(cfg) == slot_count(wl) == orc.n_slots(
        wl.persistent_cache_size, wl.frame_h, wl.frame_w, bh, bw, bt)
    for lf in range(bt, wl.window_frames + 1, bt):
        assert P.pbsa_topk_count(cfg, lf) == orc.topk_count(wl.topk_ratio, lf // bt * nbf)


def test_block344_page_sizes():
    cfg = config(WORKLOADS["decode344"])
    assert P.pbsa_blocks_per_frame(cfg) == 104        # 8 block rows (last 2 high) x 13
    assert P.pbsa_num_slots(cfg) == 208
    assert P.pbsa_topk_count(cfg, 6) == 26            # ceil(0.125 * 208)
    assert P.pbsa_topk_count(cfg, 3) == 13
    lib = P.library()
    # frame counts that are not whole 3-frame groups are rejected before any launch
    rc = lib.pbsa_select_blocks(ctypes.byref(cfg), 256, 3, 256, 4, 0, 256, 26, 256, None, 256,
                                1 << 30, None)
    assert rc == P.PBSA_ERR_ARG and "block_t" in P.pbsa_last_error()
    # a 6-frame window is not a whole number of 4-frame groups
    with pytest.raises(P.PBSAError) as e:
        P.pbsa_validate_config(config(WORKLOADS["decode"], sparse_kv_block_size=(4, 4, 4)))
    assert e.value.code == P.PBSA_ERR_ARG
    rc = lib.pbsa_cache_update(ctypes.byref(cfg), 256, 256, 6, 0, 256, 2, 0, 256, 256, 256,
                               256, 256, 256, 256, None, 0, None)
    assert rc == P.PBSA_ERR_ARG and "block_t" in P.pbsa_last_error()


def test_page_defaults_give_21_of_168():
    cfg = config(WORKLOADS["decode"])
    assert P.pbsa_blocks_per_frame(cfg) == 28
    assert P.pbsa_num_slots(cfg) == 168
    assert P.pbsa_topk_count(cfg, 6) == 21
    assert P.pbsa_topk_count(cfg, 3) == 11
    dense = config(WORKLOADS["decode"], use_local_block_sparse_attn=False)
    assert P.pbsa_topk_count(dense, 6) == 168


@pytest.mark.parametrize("field,value,code", [
    ("D", 96, P.PBSA_ERR_UNSUPPORTED),
    ("total_cache_size", 18000, P.PBSA_ERR_ARG),
    ("local_cache_size", 9000, P.PBSA_ERR_ARG),
    ("local_block_sparse_topk_ratio", 0.0, P.PBSA_ERR_ARG),
    ("local_block_sparse_topk_ratio", 1.5, P.PBSA_ERR_ARG),
    ("block_h", 9, P.PBSA_ERR_UNSUPPORTED),      # 1 x 9 x 8 = 72 tokens > 64
    ("block_t", 0, P.PBSA_ERR_ARG),
    ("kv_cache_mode", 3, P.PBSA_ERR_UNSUPPORTED),
    ("max_seq_len", 100, P.PBSA_ERR_ARG),
    ("B", 0, P.PBSA_ERR_ARG),
])
def test_invalid_configs_are_rejected(field, value, code):
    cfg = config(WORKLOADS["decode"])
    setattr(cfg, field, value)
    with pytest.raises(P.PBSAError) as e:
        P.pbsa_validate_config(cfg)
    assert e.value.code == code
    assert P.pbsa_last_error()


def test_workspace_sizes():
    cfg = config(WORKLOADS["decode"])
    # pooled means: (84 query + 168 local blocks) x 12 heads x 128 fp32
    assert P.pbsa_workspace_size(cfg, P.PBSA_OP_SELECT, 3) >= (84 + 168) * 12 * 128 * 4
    # mass partials: 42 tiles x 12 heads x (168 + 42) segments x 128 rows fp32
    assert P.pbsa_workspace_size(cfg, P.PBSA_OP_FWD, 3) >= 42 * 12 * 210 * 128 * 4
    assert P.pbsa_workspace_size(cfg, P.PBSA_OP_BWD, 3) >= 12 * 4680 * 4


def test_argument_errors_are_reported_before_any_launch():
    cfg = config(WORKLOADS["decode"])
    lib = P.library()
    # NULL query
    rc = lib.pbsa_select_blocks(ctypes.byref(cfg), None, 3, 256, 6, 0, 256, 21, 256, None,
                                256, 1 << 20, None)
    assert rc == P.PBSA_ERR_ARG and "q is NULL" in P.pbsa_last_error()
    # misaligned pointer
    rc = lib.pbsa_select_blocks(ctypes.byref(cfg), 258, 3, 256, 6, 0, 256, 21, 256, None,
                                256, 1 << 20, None)
    assert rc == P.PBSA_ERR_ARG and "aligned" in P.pbsa_last_error()
    # window larger than the ring, bad ring head, chunk beyond max_seq_len
    for args in [(3, 7, 0), (3, 6, 6), (22, 6, 0)]:
        qf, lf, rh = args
        rc = lib.pbsa_select_blocks(ctypes.byref(cfg), 256, qf, 256, lf, rh, 256, 21, 256,
                                    None, 256, 1 << 30, None)
        assert rc == P.PBSA_ERR_ARG, args
    # idx_stride smaller than k
    rc = lib.pbsa_select_blocks(ctypes.byref(cfg), 256, 3, 256, 6, 0, 256, 20, 256, None,
                                256, 1 << 30, None)
    assert rc == P.PBSA_ERR_ARG and "idx_stride" in P.pbsa_last_error()
    # workspace too small
    rc = lib.pbsa_select_blocks(ctypes.byref(cfg), 256, 3, 256, 6, 0, 256, 21, 256, None,
                                256, 16, None)
    assert rc == P.PBSA_ERR_WORKSPACE
    # cache update evicting more frames than the window holds
    rc = lib.pbsa_cache_update(ctypes.byref(cfg), 256, 256, 3, 0, 256, 4, 0, 256, 256, 256,
                               256, 256, 256, 256, None, 0, None)
    assert rc == P.PBSA_ERR_ARG and "n_evict_frames" in P.pbsa_last_error()


def test_dense_cache_mode_queries():
    wl = WORKLOADS["decode"]
    cfg = config(wl, kv_cache_mode="dense")
    P.pbsa_validate_config(cfg)
    W, S, _ = orc.cache_geometry("dense", wl.total_cache_size, wl.local_cache_size,
                                 wl.persistent_cache_size, wl.frame_h, wl.frame_w)
    assert P.pbsa_window_frames(cfg) == W == 12
    assert P.pbsa_num_slots(cfg) == S == 0
    assert P.pbsa_topk_count(cfg, 12) == 12 * 28          # every block of the window
    assert P.pbsa_workspace_size(cfg, P.PBSA_OP_FWD, 3) > 0
    bad = config(wl, kv_cache_mode="dense")
    bad.total_cache_size, bad.persistent_cache_size = 18720 + 100, 9360 + 100
    with pytest.raises(P.PBSAError) as e:
        P.pbsa_validate_config(bad)
    assert e.value.code == P.PBSA_ERR_ARG
