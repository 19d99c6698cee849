#!/usr/bin/env python
"""Benchmark of the PBSA hot path on the page-sized decode step.

Workload (Sparse Forcing project page, usage snippet sizes): B=1, 12 heads, head dim 128,
30x52-token frames, local window 9360 tokens (6 frames, 168 blocks), persistent cache
9360 tokens (168 slots), 3-frame query chunk (84 query blocks), top-0.125 (k = 21).

One step = one pass of the whole hot path over one chunk (the t=0 KV pass of the
pith.science algorithm fragment, plus the gradient of that pass):
    append the chunk's frames (ring + key means) -> select (pool Q + score + top-k)
    -> forward with block mass -> backward (dO random) -> window slide + persistent merge
Every timed step works on its own cache set (~140 MB of caches and queries), so the data a
step reads is not in the 126 MB L2 from an earlier step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload decode|sweep|train]
Prints one JSON line on rank 0.  --workload sweep runs the long-horizon decode sweep
(persistent x local x ratio x batch, 60 chunks per point, with torch's dense attention at
the same shapes) and --workload train the 21-frame training forward + backward; each prints
its own JSON line (the headline line is the decode workload's).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_35_b200.synth import WORKLOADS, block_extents, decode_inputs  # noqa: E402

WL = WORKLOADS["decode"]
METRIC = "PBSA effective TFLOP/s per decode chunk (append + select + fwd/mass + bwd + slide/merge)"
UNIT = "TFLOP/s"
WORKLOAD_NAME = ("decode chunk: B1 H12 D128, 30x52 frames, local 9360 tok (6 fr, 168 blk), "
                 "persistent 9360 tok (168 slots), chunk 3 fr (84 qblk), top-0.125 (k=21)")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "sweep", "train"])
    ap.add_argument("--no-bwd", action="store_true", help="time append/select/fwd/slide only")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-attention comparison")
    ap.add_argument("--no-344", action="store_true", help="skip the [3,4,4] block-size step")
    return ap.parse_args()
# ----------------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    """One process per GPU (torchrun env); NCCL on GPUs, gloo where there is none (the
    host-side logic is exercised that way on CPU)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def _reduce_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def all_max(ws, x):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_sum(ws, x):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------------- clocks
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9]
        mx = [float(r[2]) for r in rows if len(r) >= 9]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            if len(r) < 9:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip() == "Active":
                    reasons.add(n)
        load = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------- FLOP count
def keys_per_step(idx, cnt, pers_len, qblock_ids=None, wl=WL):
    """Sum over query tokens of the keys each attends to (valid tokens only).  idx/cnt
    cover the query blocks `qblock_ids` (all of the chunk when None)."""
    bt, bh, bw = wl.block
    ext = block_extents(wl.frame_h, wl.frame_w, bh, bw)
    sizes = torch.tensor([bt * r * c for r, c in ext], dtype=torch.int64)
    nbf = len(ext)
    idx = idx.long().cpu()
    cnt = cnt.long().cpu()
    pl = pers_len.long().cpu()
    B, H, QB, K = idx.shape
    pers_tok = pl.sum(-1)                                   # [B, H]
    valid = torch.arange(K)[None, None, None, :] < cnt[..., None]
    loc = (sizes[idx.clamp(min=0) % nbf] * valid).sum(-1)   # [B, H, QB] local keys
    qids = torch.arange(QB) if qblock_ids is None else qblock_ids
    qsz = sizes[qids % nbf]                                 # query block sizes
    return int(((pers_tok[..., None] + loc) * qsz).sum())


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops", 1590.0), d.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


# -------------------------------------------------------------------- CPU oracle
def oracle_sample(seed_offset=0, heads=1, qblocks=None):
    """The oracle (as it stands) on a sample of the decode step: `heads` heads, and of each
    head the query blocks `qblocks` (all when None): select, forward with mass, backward,
    merge.  Returns (seconds, algorithmic FLOPs of the sample, threads)."""
    import numpy as np
    from oracle import pbsa_oracle as orc
    inp = decode_inputs(WL, seed=WL.seed + seed_offset)
    f64 = lambda t: t.to(torch.float64).numpy()
    q = f64(inp["q"][:, :, :heads])
    kl = f64(inp["k_local"][:, :, :heads])
    vl = f64(inp["v_local"][:, :, :heads])
    kp = f64(inp["k_pers"][:, :heads])
    vp = f64(inp["v_pers"][:, :heads])
    pl = inp["pers_len"][:, :heads].numpy()
    dO = np.random.default_rng(seed_offset).standard_normal(q.shape)
    t0 = time.perf_counter()
    idx, _ = orc.select_blocks(q, kl, WL.frame_h, WL.frame_w, WL.topk_ratio)
    hl = [(0, h) for h in range(heads)]
    O, lse, mp, ml = orc.attn_fwd(q, kp, vp, pl, kl, vl, idx, WL.frame_h, WL.frame_w,
                                  heads=hl, qblocks=qblocks)
    orc.attn_bwd(q, kp, vp, pl, kl, vl, idx, dO, WL.frame_h, WL.frame_w, qblocks=qblocks)
    orc.cache_update(kp, vp, pl, mp, np.full(pl.shape, -1), kl, vl, ml, 3, 0,
                     WL.frame_h, WL.frame_w)
    dt = time.perf_counter() - t0
    sel = torch.from_numpy(idx)
    if qblocks is not None:
        sel = sel[:, :, qblocks]
    cnt = torch.full(sel.shape[:3], sel.shape[-1], dtype=torch.int32)
    keys = keys_per_step(sel, cnt, torch.from_numpy(pl),
                         qblock_ids=None if qblocks is None else torch.tensor(qblocks))
    flops = 14 * WL.D * keys
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count()
    return dt, flops, threads


def run_reference(args, ws, rank):
    if rank != 0:
        return
    times, flops = [], []
    for s in range(args.warmup + args.steps):
        dt, fl, threads = oracle_sample(seed_offset=s % 2, heads=1, qblocks=list(range(28)))
        if s >= args.warmup:
            times.append(dt)
            flops.append(fl)
    tot_t = sum(times)
    value = sum(flops) / tot_t / 1e12
    sample = ("per step: 1 of 12 heads, 28 of 84 query blocks (one frame) of the decode chunk: "
              "select + forward with mass + backward + merge")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD_NAME, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------------------------------ our path
def make_sets(n, dev, with_bwd, wl=WL):
    """n cache sets at the start of a chunk: the window holds its W - E oldest frames (ring
    + key means), the persistent cache is full, and the chunk's queries, its E new frames'
    keys/values and (for the backward) dO are on the device."""
    from block_sparse_attention_35_b200.attention import SparseForcingAttention
    sets = []
    shared = None
    tf, E = wl.tokens_per_frame, wl.q_frames
    for s in range(n):
        a = SparseForcingAttention(wl.B, wl.H, wl.D, wl.frame_h, wl.frame_w,
                                   wl.total_cache_size, wl.local_cache_size,
                                   wl.persistent_cache_size, sparse_kv_block_size=wl.block,
                                   max_seq_len=wl.max_seq_len,
                                   local_block_sparse_topk_ratio=wl.topk_ratio,
                                   chunk_frames=E, device=dev)
        if shared is None:
            if with_bwd:   # gradient outputs, allocated once, outside any timed region
                a.backward_buffers()
            shared = (a.ws_select, a.ws_fwd, a.ws_bwd, a._grads)
        else:
            a.ws_select, a.ws_fwd, a.ws_bwd, a._grads = shared
        inp = decode_inputs(wl, seed=wl.seed + 100 + s)
        keep = (a.W - E) * tf
        a.k_local[:, :keep].copy_(inp["k_local"][:, :keep])
        a.v_local[:, :keep].copy_(inp["v_local"][:, :keep])
        a.local_frames = a.W - E
        a.frames_seen = a.W - E
        a.pool_window()
        a.load_persistent(inp["k_pers"], inp["v_pers"], inp["pers_len"])
        k_new = inp["k_local"][:, keep:].to(dev)
        v_new = inp["v_local"][:, keep:].to(dev)
        q = inp["q"].to(dev)
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(s)).to(torch.bfloat16).to(dev) \
            if with_bwd else None
        sets.append((a, q, k_new, v_new, dout))
    return sets


def step(a, q, k_new, v_new, dout, ev=None):
    """One pass of the hot path; `ev` (list of 6 events) brackets append/select/fwd/bwd/slide."""
    if ev:
        ev[0].record()
    a.append(k_new, v_new)
    if ev:
        ev[1].record()
    a.select(q)
    if ev:
        ev[2].record()
    a.attend(q, accumulate_mass=True)
    if ev:
        ev[3].record()
    if dout is not None:
        a.backward(q, dout)
    if ev:
        ev[4].record()
    a.slide()
    if ev:
        ev[5].record()


def kernels_per_step(with_bwd):
    # append, pool (queries), score/top-k, forward, [delta, dQ + dK/dV grid], merge rank, merge copy
    return 6 + (2 if with_bwd else 0)


def bwd_available(dev):
    from block_sparse_attention_35_b200 import pbsa as P
    from block_sparse_attention_35_b200.attention import SparseForcingAttention
    a = SparseForcingAttention(1, 1, 64, 8, 8, 192, 128, 64, max_seq_len=256,
                               local_block_sparse_topk_ratio=0.5, chunk_frames=1, device=dev)
    q = torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16, device=dev)
    a.append(q, q)
    a(q)
    try:
        a.backward(q, q)
        torch.cuda.synchronize()
        return True
    except P.PBSAError as e:
        if e.code == P.PBSA_ERR_UNSUPPORTED:
            return False
        raise


def time_steps(args, sets, with_bwd, ws, wl=WL, clocks=None):
    """Warm-up, then args.steps timed steps (one cache set each) between a barrier and a
    synchronize on both sides; returns the times and exact FLOP counts."""
    n_sets = len(sets)
    for w in range(args.warmup):
        a, q, k_new, v_new, do = sets[w % n_sets]
        step(a, q, k_new, v_new, do)
    torch.cuda.synchronize()
    # exact FLOPs: each timed step uses its own set; snapshot persistent lengths first
    plens = [a.pers_len.clone() for a, *_ in sets]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    if clocks:
        clocks.start()
    barrier(ws)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for s in range(args.steps):
        a, q, k_new, v_new, do = sets[s]
        step(a, q, k_new, v_new, do, evs[s])
    t1.record()
    torch.cuda.synchronize()
    barrier(ws)
    ck = clocks.stop() if clocks else None
    ms = all_max(ws, t0.elapsed_time(t1))
    keys = [keys_per_step(a.idx, a.cnt, plens[s], wl=wl) for s, (a, *_) in enumerate(sets[:args.steps])]
    fwd_flops = [4 * wl.D * k for k in keys]
    bwd_flops = [10 * wl.D * k for k in keys] if with_bwd else [0] * len(keys)
    part = lambda i: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / len(evs)
    parts = {"append": part(0), "select": part(1), "fwd": part(2),
             "bwd": part(3) if with_bwd else None, "slide_merge": part(4)}
    return ms, fwd_flops, bwd_flops, parts, ck


def run_ours(args, ws, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    with_bwd = (not args.no_bwd) and bwd_available(dev)
    sets = make_sets(args.steps, dev, with_bwd)
    torch.cuda.synchronize()
    ms, fwd_flops, bwd_flops, parts, ck = time_steps(args, sets, with_bwd, ws, clocks=Clocks(local))
    flops_all = all_sum(ws, sum(fwd_flops) + sum(bwd_flops))
    value = flops_all / (ms * 1e-3) / 1e12
    peak_tf, peak_bw, peak_src = peaks()
    fwd_avg = parts["fwd"]
    fwd_ach = (sum(fwd_flops) / len(fwd_flops)) / (fwd_avg * 1e-3) / 1e12
    dominant = {"kernel": "attn_fwd", "achieved": fwd_ach, "ms": fwd_avg}
    if with_bwd:
        bwd_avg = parts["bwd"]
        bwd_ach = (sum(bwd_flops) / len(bwd_flops)) / (bwd_avg * 1e-3) / 1e12
        if bwd_avg > fwd_avg:
            dominant = {"kernel": "attn_bwd (delta + key-tile grid)", "achieved": bwd_ach, "ms": bwd_avg}
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        traffic = json.load(open(tfile)).get(dominant["kernel"].split()[0])

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, sets, dev, with_bwd, ws)
    b344 = None
    if not args.no_344:
        b344 = run_block344(args, dev, with_bwd, ws)
    del sets
    torch.cuda.empty_cache()

    cpu = cpu1 = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        dt, fl, threads = oracle_sample(heads=2)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"2 of 12 heads of the decode chunk: select + forward with mass + "
                         f"backward + merge ({dt:.1f} s)"}
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                dt1, fl1, _ = oracle_sample(heads=1)
            cpu1 = {"value": fl1 / dt1 / 1e12, "unit": UNIT, "cores": 1, "kind": "oracle",
                    "sample": f"1 of 12 heads of the decode chunk, one thread ({dt1:.1f} s)"}
        except ImportError:
            cpu1 = None
    dense = None
    if rank == 0 and not args.no_dense:
        dense = run_dense(dev)
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAME,
                       "path": "append+select+fwd(mass)" + ("+bwd" if with_bwd else "") + "+slide/merge",
                       "l2": "inputs larger than L2: every timed step reads its own ~140 MB input set",
                       "parallelism": f"replicas x{ws} (heads/chunks independent, no collective)",
                       "timing": "mean over the timed steps (one CUDA-event pair around all of them)"},
            "kernels_ms": parts,
            "roofline": {"bound": "tensor", "kernel": dominant["kernel"],
                         "achieved": dominant["achieved"], "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": dominant["achieved"] / peak_tf, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 burst"},
            "roofline_fwd": {"bound": "tensor", "kernel": "attn_fwd (with block mass)",
                             "achieved": fwd_ach, "peak": peak_tf, "unit": "TFLOP/s",
                             "frac": fwd_ach / peak_tf, "ms": fwd_avg},
            "block_344": b344,
            "dense": dense,
            "cpu_baseline": cpu,
            "cpu_baseline_1thread": cpu1,
            "clocks": ck,
            "e2e": e2e,
            "gpu_launches": kernels_per_step(with_bwd) * args.steps,
        }
        print(json.dumps(out))


def run_block344(args, dev, with_bwd, ws):
    """The same step with the project page's [3,4,4] blocks (3 frames x 4 x 4 tokens; 104
    blocks per 3-frame group, 208 slots, k = 26): device time and TFLOP/s."""
    wl = WORKLOADS["decode344"]
    n = max(3, min(args.steps, 10))
    sub = argparse.Namespace(**{**vars(args), "steps": n, "warmup": min(args.warmup, 3)})
    sets = make_sets(n, dev, with_bwd, wl)
    ms, ff, bf, parts, _ = time_steps(sub, sets, with_bwd, ws, wl=wl)
    peak_tf, _, _ = peaks()
    flops = all_sum(ws, sum(ff) + sum(bf))
    fwd_ach = (sum(ff) / len(ff)) / (parts["fwd"] * 1e-3) / 1e12
    out = {"workload": "decode chunk, [3,4,4] blocks: 104 blocks / 3 frames, 208 slots, 208 window "
                       "blocks, k=26", "steps": n, "ms_per_step": ms / n,
           "tflops": flops / (ms * 1e-3) / 1e12, "kernels_ms": parts,
           "fwd_tflops": fwd_ach, "fwd_frac": fwd_ach / peak_tf}
    if with_bwd:
        out["bwd_tflops"] = (sum(bf) / len(bf)) / (parts["bwd"] * 1e-3) / 1e12
        out["bwd_frac"] = out["bwd_tflops"] / peak_tf
    del sets
    return out


def _time_ms(fn, reps=10, warm=3):
    for _ in range(warm):
        fn()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(reps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / reps


def _dense_inputs(a, q, wl):
    """torch layouts of the query chunk and the whole cache (every persistent slot row and
    every window token) for the dense comparison."""
    qd = q.permute(0, 2, 1, 3).contiguous()                                # [B, H, Nq, D]
    kp = a.k_pers.reshape(wl.B, wl.H, -1, wl.D)                            # [B, H, S*64, D]
    kd = torch.cat([kp, a.k_local.permute(0, 2, 1, 3)], dim=2).contiguous()
    vp = a.v_pers.reshape(wl.B, wl.H, -1, wl.D)
    vd = torch.cat([vp, a.v_local.permute(0, 2, 1, 3)], dim=2).contiguous()
    return qd, kd, vd


def run_dense(dev):
    """The dense comparison at the same shapes on the same GPU: torch's scaled-dot-product
    attention (bf16, its flash kernel) over the whole cache (every persistent slot row and
    every window token), the PBSA forward at ratio 1 (every local block selected), and the
    PBSA forward at the workload's ratio, the last two without block mass.  Warm L2, 10
    launches each."""
    from block_sparse_attention_35_b200.attention import SparseForcingAttention
    (a, q, k_new, v_new, _), = make_sets(1, dev, False)
    a.append(k_new, v_new)
    nq = q.shape[1]
    qd, kd, vd = _dense_inputs(a, q, WL)
    nk = kd.shape[2]
    sdpa = torch.nn.functional.scaled_dot_product_attention
    sdpa_ms = _time_ms(lambda: sdpa(qd, kd, vd))
    qg = qd.clone().requires_grad_(True)
    kg = kd.clone().requires_grad_(True)
    vg = vd.clone().requires_grad_(True)
    go = torch.randn_like(qd)

    def fb():
        o = sdpa(qg, kg, vg)
        o.backward(go)
    sdpa_fb_ms = _time_ms(fb)
    a.select(q)
    pbsa_ms = _time_ms(lambda: a.attend(q, accumulate_mass=False))
    a1 = SparseForcingAttention(WL.B, WL.H, WL.D, WL.frame_h, WL.frame_w, WL.total_cache_size,
                                WL.local_cache_size, WL.persistent_cache_size,
                                max_seq_len=WL.max_seq_len, local_block_sparse_topk_ratio=1.0,
                                chunk_frames=WL.q_frames, device=dev)
    a1.k_local.copy_(a.k_local)
    a1.v_local.copy_(a.v_local)
    a1.local_frames = a1.W
    a1.pool_window()
    a1.load_persistent(a.k_pers, a.v_pers, a.pers_len)
    a1.select(q)
    ratio1_ms = _time_ms(lambda: a1.attend(q, accumulate_mass=False))
    dense_fl = 4.0 * WL.D * nq * nk * WL.H
    return {"sdpa_fwd_ms": sdpa_ms, "sdpa_fwd_bwd_ms": sdpa_fb_ms,
            "sdpa_fwd_tflops": dense_fl / (sdpa_ms * 1e-3) / 1e12,
            "pbsa_fwd_ms": pbsa_ms, "pbsa_ratio1_fwd_ms": ratio1_ms,
            "keys_dense": nk, "note": "forward without block mass; warm L2; sdpa keys include "
                                      "the persistent slots' padding rows"}


def run_e2e(args, sets, dev, with_bwd, ws):
    """The same steps through the public API (SparseForcingAttention) with every step's
    inputs (Q, the new frames' K and V, dO) copied from pinned host memory and the output O
    read back.  Copies run on a separate stream with double-buffered host and device
    staging, so step s+1's uploads and step s's download overlap the kernels; the timed
    region starts before the first upload and ends after the last download.  FLOPs are
    counted from the selections of these steps."""
    tf = WL.tokens_per_frame
    chunk = (WL.B, WL.q_frames * tf, WL.H, WL.D)
    g = torch.Generator().manual_seed(7)
    names = ["q", "k", "v"] + (["do"] if with_bwd else [])
    host = [{n: torch.randn(chunk, generator=g).to(torch.bfloat16).pin_memory() for n in names}
            for _ in range(2)]
    hout = [torch.empty(chunk, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    stage = [{n: torch.empty(chunk, dtype=torch.bfloat16, device=dev) for n in names} for _ in range(2)]
    ostage = [torch.empty(chunk, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_used = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]

    def upload(s):
        b = s % 2
        with torch.cuda.stream(copy):
            if s >= 2:
                copy.wait_event(ev_used[b])          # step s-2 has consumed this staging
            for n in names:
                stage[b][n].copy_(host[b][n], non_blocking=True)
            ev_in[b].record(copy)

    def compute(s, a, record):
        b = s % 2
        comp.wait_event(ev_in[b])
        st = stage[b]
        a.append(st["k"], st["v"])
        a.select(st["q"])
        a.attend(st["q"], accumulate_mass=True)
        if with_bwd:
            a.backward(st["q"], st["do"])
        if s >= 2:
            comp.wait_event(ev_done[b])              # the download of step s-2 has finished
        ostage[b].copy_(a.out)
        ev_used[b].record(comp)
        ev_out[b].record(comp)
        if record is not None:
            record.append((a.idx.clone(), a.cnt.clone(), a.pers_len.clone()))
        a.slide()
        with torch.cuda.stream(copy):
            copy.wait_event(ev_out[b])
            hout[b].copy_(ostage[b], non_blocking=True)
            ev_done[b].record(copy)

    def run(n, record=None):
        upload(0)
        for s in range(n):
            if s + 1 < n:
                upload(s + 1)
            compute(s, sets[s % len(sets)][0], record)

    run(args.warmup)
    torch.cuda.synchronize()
    barrier(ws)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    copy.wait_event(t0)
    rec = []
    run(args.steps, rec)
    comp.wait_stream(copy)
    t1.record(comp)
    torch.cuda.synchronize()
    ms = all_max(ws, t0.elapsed_time(t1))
    keys = [keys_per_step(i, c, p) for i, c, p in rec]
    flops = all_sum(ws, sum((14 if with_bwd else 4) * WL.D * k for k in keys))
    h2d = sum(host[0][n].numel() * 2 for n in names)
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": hout[0].numel() * 2, "ms_per_step": ms / args.steps,
            "copies": "copy stream, double-buffered pinned host and device staging"}


# ------------------------------------------------------------- long-horizon sweep
def run_sweep(args, ws, rank, local):
    """Long-horizon decode sweep: persistent cache {4680, 9360, 18720} tokens x local window
    {4680, 9360} x top-k ratio {1/16, 1/8, 1/4} x batch {1, 4}, 60 chunks per point (append
    -> select -> forward with mass -> slide/merge, steady-state caches), and torch's dense
    attention over the same whole cache as the comparison."""
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peak_tf, _, _ = peaks()
    chunks = 60
    rows = []
    for P_tok in (4680, 9360, 18720):
        for L_tok in (4680, 9360):
            for ratio in (1 / 16, 1 / 8, 1 / 4):
                for B in (1, 4):
                    wl = dataclasses.replace(WL, B=B, persistent_cache_size=P_tok,
                                             local_cache_size=L_tok, total_cache_size=P_tok + L_tok,
                                             topk_ratio=ratio, seed=60)
                    (a, q, k_new, v_new, _), = make_sets(1, dev, False, wl)
                    for _ in range(3):
                        step(a, q, k_new, v_new, None)
                    torch.cuda.synchronize()
                    plen = a.pers_len.clone()
                    t0 = torch.cuda.Event(enable_timing=True)
                    t1 = torch.cuda.Event(enable_timing=True)
                    t0.record()
                    for _ in range(chunks):
                        step(a, q, k_new, v_new, None)
                    t1.record()
                    torch.cuda.synchronize()
                    ms = t0.elapsed_time(t1) / chunks
                    keys = keys_per_step(a.idx, a.cnt, plen, wl=wl)
                    a.append(k_new, v_new)
                    a.select(q)
                    fwd_ms = _time_ms(lambda: a.attend(q, accumulate_mass=True))
                    qd, kd, vd = _dense_inputs(a, q, wl)
                    sdpa_ms = _time_ms(lambda: torch.nn.functional.scaled_dot_product_attention(qd, kd, vd))
                    fl = 4 * wl.D * keys
                    rows.append({"persistent": P_tok, "local": L_tok, "ratio": ratio, "B": B,
                                 "k": int(a.kmax), "chunk_ms": ms, "fwd_ms": fwd_ms,
                                 "fwd_tflops": fl / (fwd_ms * 1e-3) / 1e12,
                                 "fwd_frac": fl / (fwd_ms * 1e-3) / 1e12 / peak_tf,
                                 "sdpa_fwd_ms": sdpa_ms, "dense_keys": kd.shape[2],
                                 "speedup_vs_sdpa": sdpa_ms / fwd_ms})
                    del a, q, k_new, v_new, qd, kd, vd
                    torch.cuda.empty_cache()
    if rank == 0:
        tot = sum(r["chunk_ms"] for r in rows)
        print(json.dumps({"metric": "PBSA ms per decode chunk over the long-horizon sweep",
                          "value": tot / len(rows), "unit": "ms/chunk (mean over points)",
                          "higher_is_better": False, "n_gpus": ws, "dtype": "bf16",
                          "data": "synthetic", "config": {"workload": "sweep", "chunks_per_point": chunks,
                                                          "chunk": "append + select + fwd(mass) + slide/merge"},
                          "points": rows}))


# ----------------------------------------------------------------------- training
def run_train(args, ws, rank, local):
    """Training forward + backward over the 21-frame sequence (32 760 tokens): 7 chunk-causal
    chunks of 3 frames, each over a synthetic persistent cache of 168 slots (9360 tokens)
    and a top-0.125 selection over its (at most 6-frame) window: k = 11 for chunk 0 (84
    blocks), 21 after.  Compared with torch's dense attention of each chunk over every
    earlier frame plus the persistent rows (what the chunk would attend without sparsity)."""
    from block_sparse_attention_35_b200.attention import SparseForcingAttention
    from block_sparse_attention_35_b200.synth import training_inputs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = WORKLOADS["train"]
    tf, E, W = wl.tokens_per_frame, wl.q_frames, wl.window_frames
    inp = training_inputs(wl)
    a = SparseForcingAttention(wl.B, wl.H, wl.D, wl.frame_h, wl.frame_w, wl.total_cache_size,
                               wl.local_cache_size, wl.persistent_cache_size,
                               max_seq_len=wl.max_seq_len, local_block_sparse_topk_ratio=wl.topk_ratio,
                               chunk_frames=E, device=dev)
    a.backward_buffers()
    a.load_persistent(inp["k_pers"], inp["v_pers"], inp["pers_len"])
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    plen = a.pers_len.clone()

    def chunk_views(c):
        sl = slice(c * E * tf, (c + 1) * E * tf)
        return q[:, sl], k[:, sl], v[:, sl], do[:, sl]

    def one_pass(record=None):
        a.ring_head, a.local_frames, a.frames_seen, a.first_frame_global = 0, 0, 0, 0
        for c in range(wl.chunks):
            qc, kc, vc, dc = chunk_views(c)
            if a.local_frames + E > W:
                a.ring_head = (a.ring_head + E) % W      # chunk-causal window: drop the oldest chunk
                a.local_frames -= E
                a.first_frame_global += E
            a.append(kc, vc)
            a.select(qc)
            a.attend(qc)
            a.backward(qc, dc)
            if record is not None:
                record.append((a.idx.clone(), a.cnt.clone()))

    for _ in range(max(2, args.warmup)):
        one_pass()
    torch.cuda.synchronize()
    reps = 5
    rec = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for r in range(reps):
        one_pass(rec if r == 0 else None)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / reps
    keys = sum(keys_per_step(i, c, plen, wl=wl) for i, c in rec)
    flops = 14 * wl.D * keys
    # dense: chunk c attends (every persistent row +) every frame up to its end
    kp = a.k_pers.reshape(wl.B, wl.H, -1, wl.D)
    vp = a.v_pers.reshape(wl.B, wl.H, -1, wl.D)
    sdpa = torch.nn.functional.scaled_dot_product_attention
    tot_fb = 0.0
    for c in range(wl.chunks):
        sl = slice(c * E * tf, (c + 1) * E * tf)
        qd = q[:, sl].permute(0, 2, 1, 3).contiguous().requires_grad_(True)
        kd = torch.cat([kp, k[:, :(c + 1) * E * tf].permute(0, 2, 1, 3)], 2).contiguous().requires_grad_(True)
        vd = torch.cat([vp, v[:, :(c + 1) * E * tf].permute(0, 2, 1, 3)], 2).contiguous().requires_grad_(True)
        go = do[:, sl].permute(0, 2, 1, 3).contiguous()

        def fb():
            sdpa(qd, kd, vd).backward(go)
        tot_fb += _time_ms(fb, reps=5, warm=2)
    peak_tf, _, _ = peaks()
    if rank == 0:
        print(json.dumps({"metric": "PBSA training forward+backward over 21 frames (32760 tokens)",
                          "value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "higher_is_better": True,
                          "ms": ms, "frac": flops / (ms * 1e-3) / 1e12 / peak_tf,
                          "tflop": flops / 1e12, "n_gpus": ws, "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": "train: B1 H12 D128, 21 frames in 7 chunks of 3, "
                                                 "168 persistent slots, top-0.125 over a <=6-frame window",
                                     "step": "per chunk: append + select + fwd + bwd"},
                          "dense_chunk_causal_fwd_bwd_ms": tot_fb}))


def main():
    args = parse()
    ws, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        elif args.workload == "sweep":
            run_sweep(args, ws, rank, local)
        elif args.workload == "train":
            run_train(args, ws, rank, local)
        else:
            run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
