#!/usr/bin/env python
"""Benchmark of the PBSA hot path on the page-sized decode step.

Workload (Sparse Forcing project page, usage snippet sizes): B=1, 12 heads, head dim 128,
30x52-token frames, local window 9360 tokens (6 frames, 168 blocks), persistent cache
9360 tokens (168 slots), 3-frame query chunk (84 query blocks), top-0.125 (k = 21).

One step = one pass of the whole hot path over one chunk:
    select (pool + score + top-k) -> forward with block mass -> backward (dO random)
    -> window slide + persistent merge
(the t=0 KV pass of the pith.science algorithm fragment, plus the gradient of that pass).
Every timed step works on its own input set (~140 MB of caches and queries), so the data a
step reads is not in the 126 MB L2 from an earlier step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
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
METRIC = "PBSA effective TFLOP/s per decode chunk (select + fwd/mass + bwd + slide/merge)"
UNIT = "TFLOP/s"
WORKLOAD_NAME = ("decode chunk: B1 H12 D128, 30x52 frames, local 9360 tok (6 fr, 168 blk), "
                 "persistent 9360 tok (168 slots), chunk 3 fr (84 qblk), top-0.125 (k=21)")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-bwd", action="store_true", help="time select/fwd/slide only")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-attention comparison")
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
def keys_per_step(idx, cnt, pers_len, qblock_ids=None):
    """Sum over query tokens of the keys each attends to (valid tokens only).  idx/cnt
    cover the query blocks `qblock_ids` (all of the chunk when None)."""
    ext = block_extents(WL.frame_h, WL.frame_w)
    sizes = torch.tensor([r * c for r, c in ext], dtype=torch.int64)
    nbf = len(ext)
    idx = idx.long().cpu()
    cnt = cnt.long().cpu()
    pl = pers_len.long().cpu()
    B, H, QB, K = idx.shape
    pers_tok = pl.sum(-1)                                   # [B, H]
    valid = torch.arange(K)[None, None, None, :] < cnt[..., None]
    loc = (sizes[idx % nbf] * valid).sum(-1)                # [B, H, QB] local keys
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
def make_sets(n, dev, with_bwd):
    from block_sparse_attention_35_b200.attention import SparseForcingAttention
    sets = []
    shared = None
    for s in range(n):
        a = SparseForcingAttention(WL.B, WL.H, WL.D, WL.frame_h, WL.frame_w,
                                   WL.total_cache_size, WL.local_cache_size,
                                   WL.persistent_cache_size, max_seq_len=WL.max_seq_len,
                                   local_block_sparse_topk_ratio=WL.topk_ratio,
                                   chunk_frames=WL.q_frames, device=dev)
        if shared is None:
            if with_bwd:   # gradient outputs, allocated once, outside any timed region
                a.backward_buffers()
            shared = (a.ws_select, a.ws_fwd, a.ws_bwd, a._grads)
        else:
            a.ws_select, a.ws_fwd, a.ws_bwd, a._grads = shared
        inp = decode_inputs(WL, seed=WL.seed + 100 + s)
        a.k_local.copy_(inp["k_local"])
        a.v_local.copy_(inp["v_local"])
        a.local_frames = a.W
        a.load_persistent(inp["k_pers"], inp["v_pers"], inp["pers_len"])
        q = inp["q"].to(dev)
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(s)).to(torch.bfloat16).to(dev) \
            if with_bwd else None
        sets.append((a, q, dout))
    return sets


def step(a, q, dout, ev=None):
    """One pass of the hot path; `ev` (list of 5 events) brackets select/fwd/bwd/slide."""
    if ev:
        ev[0].record()
    a.select(q)
    if ev:
        ev[1].record()
    a.attend(q, accumulate_mass=True)
    if ev:
        ev[2].record()
    if dout is not None:
        a.backward(q, dout)
    if ev:
        ev[3].record()
    a.slide(WL.q_frames)
    if ev:
        ev[4].record()
    a.local_frames = a.W  # the freed slots now hold the next chunk's frames


def kernels_per_step(with_bwd):
    # pool, score/top-k, forward, [delta, dQ + dK/dV grid], merge rank, merge copy
    return 5 + (2 if with_bwd else 0)


def bwd_available(dev):
    from block_sparse_attention_35_b200 import pbsa as P
    from block_sparse_attention_35_b200.attention import SparseForcingAttention
    a = SparseForcingAttention(1, 1, 64, 8, 8, 192, 128, 64, max_seq_len=256,
                               local_block_sparse_topk_ratio=0.5, chunk_frames=1, device=dev)
    a.local_frames = 1
    q = torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16, device=dev)
    a(q)
    try:
        a.backward(q, q)
        torch.cuda.synchronize()
        return True
    except P.PBSAError as e:
        if e.code == P.PBSA_ERR_UNSUPPORTED:
            return False
        raise


def run_ours(args, ws, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    with_bwd = (not args.no_bwd) and bwd_available(dev)
    n_sets = args.steps
    sets = make_sets(n_sets, dev, with_bwd)
    torch.cuda.synchronize()
    for w in range(args.warmup):
        a, q, do = sets[w % n_sets]
        step(a, q, do)
    torch.cuda.synchronize()
    # exact FLOPs: each timed step uses its own set; snapshot persistent lengths first
    plens = [a.pers_len.clone() for a, _, _ in sets]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = Clocks(local)
    clocks.start()
    barrier(ws)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for s in range(args.steps):
        a, q, do = sets[s]
        step(a, q, do, evs[s])
    t1.record()
    torch.cuda.synchronize()
    barrier(ws)
    ck = clocks.stop()
    ms_local = t0.elapsed_time(t1)
    ms = all_max(ws, ms_local)
    keys = [keys_per_step(a.idx, a.cnt, plens[s]) for s, (a, _, _) in enumerate(sets)]
    fwd_flops = [4 * WL.D * k for k in keys]
    bwd_flops = [10 * WL.D * k for k in keys] if with_bwd else [0] * len(keys)
    flops_local = sum(fwd_flops) + sum(bwd_flops)
    flops_all = all_sum(ws, flops_local)
    value = flops_all / (ms * 1e-3) / 1e12
    sel_ms = [e[0].elapsed_time(e[1]) for e in evs]
    fwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    bwd_ms = [e[2].elapsed_time(e[3]) for e in evs]
    upd_ms = [e[3].elapsed_time(e[4]) for e in evs]
    peak_tf, peak_bw, peak_src = peaks()
    fwd_avg = sum(fwd_ms) / len(fwd_ms)
    fwd_ach = (sum(fwd_flops) / len(fwd_flops)) / (fwd_avg * 1e-3) / 1e12
    dominant = {"kernel": "attn_fwd", "achieved": fwd_ach, "ms": fwd_avg}
    if with_bwd:
        bwd_avg = sum(bwd_ms) / len(bwd_ms)
        bwd_ach = (sum(bwd_flops) / len(bwd_flops)) / (bwd_avg * 1e-3) / 1e12
        if bwd_avg > fwd_avg:
            dominant = {"kernel": "attn_bwd (delta + dQ/dK/dV grid)", "achieved": bwd_ach, "ms": bwd_avg}
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        traffic = json.load(open(tfile)).get(dominant["kernel"].split()[0])

    # ---------------------------------------------------------------- end to end
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, sets, dev, with_bwd, fwd_flops, bwd_flops, ws)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        dt, fl, threads = oracle_sample(heads=2)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"2 of 12 heads of the decode chunk: select + forward with mass + "
                         f"backward + merge ({dt:.1f} s)"}
    dense = None
    if rank == 0 and not args.no_dense:
        dense = run_dense(dev, sets[0])
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAME,
                       "path": "select+fwd(mass)" + ("+bwd" if with_bwd else "") + "+slide/merge",
                       "l2": "inputs larger than L2: every timed step reads its own ~140 MB input set",
                       "parallelism": f"replicas x{ws} (heads/chunks independent, no collective)"},
            "kernels_ms": {"select": sum(sel_ms) / len(sel_ms), "fwd": fwd_avg,
                           "bwd": (sum(bwd_ms) / len(bwd_ms)) if with_bwd else None,
                           "slide_merge": sum(upd_ms) / len(upd_ms)},
            "roofline": {"bound": "tensor", "kernel": dominant["kernel"],
                         "achieved": dominant["achieved"], "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": dominant["achieved"] / peak_tf, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 burst"},
            "roofline_fwd": {"bound": "tensor", "kernel": "attn_fwd (with block mass)",
                             "achieved": fwd_ach, "peak": peak_tf, "unit": "TFLOP/s",
                             "frac": fwd_ach / peak_tf, "ms": fwd_avg},
            "dense": dense,
            "cpu_baseline": cpu,
            "clocks": ck,
            "e2e": e2e,
            "gpu_launches": kernels_per_step(with_bwd) * args.steps,
        }
        print(json.dumps(out))


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


def run_dense(dev, first_set):
    """The dense comparison at the same shapes on the same GPU: torch's scaled-dot-product
    attention (bf16, its flash kernel) over the whole cache (every persistent slot row and
    every window token, 18720 keys), the PBSA forward at ratio 1 (every local block
    selected), and the PBSA forward at the workload's ratio, the last two without block
    mass.  Warm L2, 10 launches each."""
    from block_sparse_attention_35_b200.attention import SparseForcingAttention
    a, q, _ = first_set
    nq = q.shape[1]
    qd = q.permute(0, 2, 1, 3).contiguous()                               # [B, H, Nq, D]
    kp = a.k_pers.reshape(WL.B, WL.H, -1, WL.D)                            # [B, H, S*64, D]
    kd = torch.cat([kp, a.k_local.permute(0, 2, 1, 3)], dim=2).contiguous()
    vp = a.v_pers.reshape(WL.B, WL.H, -1, WL.D)
    vd = torch.cat([vp, a.v_local.permute(0, 2, 1, 3)], dim=2).contiguous()
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
    a1.load_persistent(a.k_pers, a.v_pers, a.pers_len)
    a1.select(q)
    ratio1_ms = _time_ms(lambda: a1.attend(q, accumulate_mass=False))
    dense_fl = 4.0 * WL.D * nq * nk * WL.H
    return {"sdpa_fwd_ms": sdpa_ms, "sdpa_fwd_bwd_ms": sdpa_fb_ms,
            "sdpa_fwd_tflops": dense_fl / (sdpa_ms * 1e-3) / 1e12,
            "pbsa_fwd_ms": pbsa_ms, "pbsa_ratio1_fwd_ms": ratio1_ms,
            "keys_dense": nk, "note": "forward without block mass; warm L2; sdpa keys include "
                                      "the persistent slots' padding rows"}


def run_e2e(args, sets, dev, with_bwd, fwd_flops, bwd_flops, ws):
    """Same steps through the public API with the chunk's inputs copied from pinned host
    memory every step and the output read back."""
    tf = WL.tokens_per_frame
    chunk = (WL.B, WL.q_frames * tf, WL.H, WL.D)
    g = torch.Generator().manual_seed(7)
    hq = torch.randn(chunk, generator=g).to(torch.bfloat16).pin_memory()
    hk = torch.randn(chunk, generator=g).to(torch.bfloat16).pin_memory()
    hv = torch.randn(chunk, generator=g).to(torch.bfloat16).pin_memory()
    hdo = torch.randn(chunk, generator=g).to(torch.bfloat16).pin_memory() if with_bwd else None
    hout = torch.empty(chunk, dtype=torch.bfloat16).pin_memory()

    def e2e_step(a, q, do):
        a.slide(WL.q_frames) if a.local_frames + WL.q_frames > a.W else None
        a.append(hk, hv)
        q.copy_(hq, non_blocking=True)
        if do is not None:
            do.copy_(hdo, non_blocking=True)
        a.select(q)
        a.attend(q, accumulate_mass=True)
        if do is not None:
            a.backward(q, do)
        hout.copy_(a.out, non_blocking=True)

    for a, _, _ in sets:
        a.local_frames = a.W
    for w in range(args.warmup):
        a, q, do = sets[w % len(sets)]
        e2e_step(a, q, do)
    torch.cuda.synchronize()
    barrier(ws)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for s in range(args.steps):
        a, q, do = sets[s]
        e2e_step(a, q, do)
    t1.record()
    torch.cuda.synchronize()
    ms = all_max(ws, t0.elapsed_time(t1))
    flops = all_sum(ws, sum(fwd_flops) + sum(bwd_flops))
    h2d = hq.numel() * 2 * (3 + (1 if with_bwd else 0))
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": hout.numel() * 2, "ms_per_step": ms / args.steps}


def main():
    args = parse()
    ws, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        else:
            run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
