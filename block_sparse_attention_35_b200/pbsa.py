"""Thin Python binding of the PBSA C ABI (include/pbsa.h).

Each ``pbsa_*`` function here has the name and argument order of the C function; it only
turns torch tensors into device pointers and the current CUDA stream into ``void*``, and
raises ``PBSAError`` on a non-zero return code.  All work runs in the CUDA kernels of
``libpbsa.so``; there is no CPU fallback, and importing this module fails loudly when the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpbsa.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "pbsa.h")

PBSA_OK = 0
PBSA_ERR_ARG = -1
PBSA_ERR_UNSUPPORTED = -2
PBSA_ERR_CUDA = -3
PBSA_ERR_TIMEOUT = -4
PBSA_ERR_DEVICE_CHECK = -5
PBSA_ERR_WORKSPACE = -6
PBSA_OP_SELECT, PBSA_OP_FWD, PBSA_OP_BWD, PBSA_OP_UPDATE = 0, 1, 2, 3
PBSA_KV_CACHE_SPARSE_FORCING, PBSA_KV_CACHE_DENSE = 0, 1


class PBSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"PBSA error {code}: {msg}")
        self.code = code


class pbsa_config(ctypes.Structure):
    """Mirror of the C struct pbsa_config."""
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
        ("frame_h", ctypes.c_int), ("frame_w", ctypes.c_int),
        ("block_t", ctypes.c_int), ("block_h", ctypes.c_int), ("block_w", ctypes.c_int),
        ("total_cache_size", ctypes.c_int), ("local_cache_size", ctypes.c_int),
        ("persistent_cache_size", ctypes.c_int), ("max_seq_len", ctypes.c_int),
        ("kv_cache_mode", ctypes.c_int), ("use_local_block_sparse_attn", ctypes.c_int),
        ("local_block_sparse_topk_ratio", ctypes.c_float),
        ("sink_frames", ctypes.c_int),
    ]


def make_config(B, H, D, frame_h, frame_w, total_cache_size, local_cache_size,
                persistent_cache_size, max_seq_len, local_block_sparse_topk_ratio,
                use_local_block_sparse_attn=True, sparse_kv_block_size=(1, 8, 8),
                kv_cache_mode="sparse_forcing", sink_frames=0) -> pbsa_config:
    """Builds a pbsa_config from the SparseForcingAttention constructor arguments (plus
    sink_frames, the length of the sequence's sink)."""
    modes = {"sparse_forcing": PBSA_KV_CACHE_SPARSE_FORCING, "dense": PBSA_KV_CACHE_DENSE}
    if kv_cache_mode not in modes:
        raise PBSAError(PBSA_ERR_UNSUPPORTED, f"kv_cache_mode {kv_cache_mode!r}")
    bt, bh, bw = sparse_kv_block_size
    return pbsa_config(B, H, D, frame_h, frame_w, bt, bh, bw, total_cache_size,
                       local_cache_size, persistent_cache_size, max_seq_len,
                       modes[kv_cache_mode], int(bool(use_local_block_sparse_attn)),
                       float(local_block_sparse_topk_ratio), int(sink_frames))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_attention_35_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I = ctypes.c_int
    C = ctypes.POINTER(pbsa_config)
    sig = {
        "pbsa_validate_config": (I, [C]),
        "pbsa_blocks_per_frame": (I, [C]),
        "pbsa_window_frames": (I, [C]),
        "pbsa_num_slots": (I, [C]),
        "pbsa_sink_slots": (I, [C]),
        "pbsa_topk_count": (I, [C, I]),
        "pbsa_workspace_size": (ctypes.c_size_t, [C, I, I]),
        "pbsa_last_error": (ctypes.c_char_p, []),
        "pbsa_version": (ctypes.c_char_p, []),
        "pbsa_select_blocks": (I, [C, P, I, P, I, I, P, I, P, P, P, ctypes.c_size_t, P]),
        "pbsa_attn_fwd": (I, [C, P, I, P, P, P, P, P, I, I, P, I, P, P, P, P, P, P,
                              ctypes.c_size_t, P, P]),
        "pbsa_attn_bwd": (I, [C, P, I, P, P, P, P, P, I, I, P, I, P, P, P, P, P, P, P, P, P,
                              P, ctypes.c_size_t, P, P]),
        "pbsa_cache_update": (I, [C, P, P, I, I, P, I, I, P, P, P, P, P, P, P, P,
                                  ctypes.c_size_t, P]),
        "pbsa_wait_selftest": (I, [P, ctypes.c_longlong, P]),
        "pbsa_pool_keys": (I, [C, P, I, I, P, P]),
        "pbsa_append_frames": (I, [C, P, P, I, I, P, P, I, P, P, P, P, P, P, P]),
        "pbsa_select_blocks_pooled": (I, [C, P, I, P, I, I, P, I, P, P, P, ctypes.c_size_t, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def header_symbols(path: str = HEADER):
    """Names of the functions declared in include/pbsa.h."""
    txt = open(path).read()
    return sorted(set(re.findall(r"PBSA_API\s+[\w\s\*]+?\b(pbsa_\w+)\s*\(", txt)))


def library():
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(rc):
    if rc != PBSA_OK:
        raise PBSAError(rc, _lib.pbsa_last_error().decode())


def _cfg(cfg):
    return ctypes.byref(cfg)


# ------------------------------------------------------------------ host-only queries
def pbsa_validate_config(cfg):
    _check(_lib.pbsa_validate_config(_cfg(cfg)))


def pbsa_blocks_per_frame(cfg) -> int:
    return _lib.pbsa_blocks_per_frame(_cfg(cfg))


def pbsa_window_frames(cfg) -> int:
    return _lib.pbsa_window_frames(_cfg(cfg))


def pbsa_num_slots(cfg) -> int:
    return _lib.pbsa_num_slots(_cfg(cfg))


def pbsa_sink_slots(cfg) -> int:
    return _lib.pbsa_sink_slots(_cfg(cfg))


def pbsa_topk_count(cfg, local_frames: int) -> int:
    k = _lib.pbsa_topk_count(_cfg(cfg), local_frames)
    if k < 0:
        _check(k)
    return k


def pbsa_workspace_size(cfg, op: int, q_frames: int) -> int:
    return int(_lib.pbsa_workspace_size(_cfg(cfg), op, q_frames))


def pbsa_version() -> str:
    return _lib.pbsa_version().decode()


def pbsa_last_error() -> str:
    return _lib.pbsa_last_error().decode()


# ------------------------------------------------------------------ device calls
def pbsa_select_blocks(cfg, q, q_frames, k_local, local_frames, ring_head, idx, idx_stride,
                       cnt, scores, workspace, stream=None):
    _check(_lib.pbsa_select_blocks(
        _cfg(cfg), _ptr(q), q_frames, _ptr(k_local), local_frames, ring_head, _ptr(idx),
        idx_stride, _ptr(cnt), _ptr(scores), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream)))


def pbsa_attn_fwd(cfg, q, q_frames, k_pers, v_pers, pers_len, k_local, v_local, local_frames,
                  ring_head, idx, idx_stride, cnt, out, lse, mass_local, mass_pers, workspace,
                  status, stream=None):
    _check(_lib.pbsa_attn_fwd(
        _cfg(cfg), _ptr(q), q_frames, _ptr(k_pers), _ptr(v_pers), _ptr(pers_len),
        _ptr(k_local), _ptr(v_local), local_frames, ring_head, _ptr(idx), idx_stride,
        _ptr(cnt), _ptr(out), _ptr(lse), _ptr(mass_local), _ptr(mass_pers), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream)))


def pbsa_attn_bwd(cfg, q, q_frames, k_pers, v_pers, pers_len, k_local, v_local, local_frames,
                  ring_head, idx, idx_stride, cnt, out, lse, dout, dq, dk_pers, dv_pers,
                  dk_local, dv_local, workspace, status, stream=None):
    _check(_lib.pbsa_attn_bwd(
        _cfg(cfg), _ptr(q), q_frames, _ptr(k_pers), _ptr(v_pers), _ptr(pers_len),
        _ptr(k_local), _ptr(v_local), local_frames, ring_head, _ptr(idx), idx_stride,
        _ptr(cnt), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk_pers), _ptr(dv_pers),
        _ptr(dk_local), _ptr(dv_local), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream)))


def pbsa_cache_update(cfg, k_local, v_local, local_frames, ring_head, mass_local,
                      n_evict_frames, first_frame_global, k_pers, v_pers, pers_len, pers_score,
                      pers_src, upd, n_upd, workspace=None, stream=None):
    _check(_lib.pbsa_cache_update(
        _cfg(cfg), _ptr(k_local), _ptr(v_local), local_frames, ring_head, _ptr(mass_local),
        n_evict_frames, first_frame_global, _ptr(k_pers), _ptr(v_pers), _ptr(pers_len),
        _ptr(pers_score), _ptr(pers_src), _ptr(upd), _ptr(n_upd), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream)))


def pbsa_wait_selftest(status, timeout_ns: int, stream=None):
    _check(_lib.pbsa_wait_selftest(_ptr(status), int(timeout_ns), _stream(stream)))


def pbsa_append_frames(cfg, k_new, v_new, n_frames, first_global_frame, k_local, v_local,
                       ring_slot, kbar=None, k_pers=None, v_pers=None, pers_len=None,
                       pers_score=None, pers_src=None, stream=None):
    """Appends frames to the cache: sink frames into their slots, the others into the ring
    from ring_slot on, with their key means written to kbar (when given) in the same pass."""
    _check(_lib.pbsa_append_frames(
        _cfg(cfg), _ptr(k_new), _ptr(v_new), n_frames, first_global_frame, _ptr(k_local),
        _ptr(v_local), ring_slot, _ptr(kbar), _ptr(k_pers), _ptr(v_pers), _ptr(pers_len),
        _ptr(pers_score), _ptr(pers_src), _stream(stream)))


def pbsa_pool_keys(cfg, k_local, first_slot, n_frames, kbar, stream=None):
    """Pools the key blocks of ring slots first_slot.. (n_frames, mod W) into kbar
    [B, H, W*NB_f, D] fp32 (row = slot * NB_f + block)."""
    _check(_lib.pbsa_pool_keys(_cfg(cfg), _ptr(k_local), first_slot, n_frames, _ptr(kbar),
                               _stream(stream)))


def pbsa_select_blocks_pooled(cfg, q, q_frames, kbar, local_frames, ring_head, idx, idx_stride,
                              cnt, scores, workspace, stream=None):
    """Block selection with the window's key means read from kbar (see pbsa_pool_keys)."""
    _check(_lib.pbsa_select_blocks_pooled(
        _cfg(cfg), _ptr(q), q_frames, _ptr(kbar), local_frames, ring_head, _ptr(idx),
        idx_stride, _ptr(cnt), _ptr(scores), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _stream(stream)))


def pbsa_select_blocks_noalloc(cfg, q, q_frames, k_local, local_frames, ring_head, idx,
                               idx_stride, cnt, scores, stream=None):
    """Block selection without a workspace, for callers that cannot allocate device
    memory (the library keeps the scratch in a static device buffer; see include/pbsa.h)."""
    f = _lib.pbsa_select_blocks_noalloc
    if f.argtypes is None:
        P, I = ctypes.c_void_p, ctypes.c_int
        f.restype = I
        f.argtypes = [ctypes.POINTER(pbsa_config), P, I, P, I, I, P, I, P, P, P]
    _check(f(_cfg(cfg), _ptr(q), q_frames, _ptr(k_local), local_frames, ring_head, _ptr(idx),
             idx_stride, _ptr(cnt), _ptr(scores), _stream(stream)))
