#!/usr/bin/env python
"""Benchmark of the BSA hot path on B200.

One step = one pass of the whole path over one batch of synthetic input resident in HBM:
fused QK-RMSNorm + 3D-RoPE prologue (with block means) -> block-pooled top-r routing ->
sparse attention forward -> sparse attention backward (with the forward's routing; dO is
a fixed synthetic upstream gradient).  Default workload: the 720p refine stage (24x45x80
latent tokens padded to 24x48x80, 4x4x8 blocks, top-r 72, 32 heads x 128, bf16).

value    = effective TFLOP/s of the step on selected-block tile FLOPs (4*BS^2*D per
           selected (query block, key block) pair forward, 2.5x that backward) summed over
           all ranks / max-over-ranks step time.
e2e      = the same metric through the public pipeline API with host (pinned) raster
           inputs q, k, v, dO copied in and the raster results O, dq, dk, dv copied back
           inside the timed region, every step (O via the inverse relayout, the gradients via
           the attention backward and the prologue backward); the copies run on their own
           streams, overlapping the neighbouring steps' compute.
roofline = the attention kernel with the longest launches (timed live with CUDA events on its
           stream through the library's kernel timing) against the measured sustained
           dense bf16 tensor peak (the kernels run inside a long step), with the burst-peak
           fraction beside it.  Each kernel reports its executed GEMM-tile FLOPs and its
           algorithmic ones: the dQ pass recomputes S and dP, which the algorithmic count
           leaves out (a backward needs 5 GEMM tiles per pair, 2.5x the forward's 2).

Multi-GPU (torchrun): every rank runs an independent replica of the workload (the path
has no exchange step: routing and attention are independent per (batch, head)), so
scaling is weak; ranks meet only at the timing barriers.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, add_smooth_field, make_raster_inputs  # noqa: E402


def tile_flops(bs: int, d: int, n_pairs: int) -> float:
    return 4.0 * bs * bs * d * n_pairs


KERNEL_NAMES = {"fwd": "bsa_fwd_kernel", "bwd_dkdv": "bsa_bwd_dkdv_kernel",
                "bwd_dq": "bsa_bwd_dq_kernel"}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per unit of work, from one ncu
# capture of the kernel as it now stands on the 480p workload (365,568 pairs; the
# attention-kernel summary under profiles/ holds the figures and the commands); a unit is a
# selected block pair (fwd, dq) or a pair with a current key block (dkdv).  Traffic grows with
# the pairs a launch processes, so a full launch is scaled from it.  None = not captured for
# the kernel as it now stands.
DRAM_BYTES_PER_PAIR = {"fwd": 3998, "bwd_dkdv": 5752, "bwd_dq": 4842}


def block_token_counts(g, frames: int) -> np.ndarray:
    """Valid tokens of each block of a `frames` x grid_h x grid_w grid (blocks t-major)."""
    bt, bh, bw = g.blk
    nbt, nbh, nbw = -(-frames // bt), -(-g.grid_h // bh), -(-g.grid_w // bw)
    vt = np.minimum(bt, frames - bt * np.arange(nbt))
    vh = np.minimum(bh, g.grid_h - bh * np.arange(nbh))
    vw = np.minimum(bw, g.grid_w - bw * np.arange(nbw))
    return (vt[:, None, None] * vh[None, :, None] * vw[None, None, :]).reshape(-1)


def valid_token_flops(g, idx: np.ndarray, cnt: np.ndarray) -> float:
    """Forward FLOPs counting valid tokens only: sum over selected pairs of 4 D n_i n_j."""
    nq = block_token_counts(g, g.t_frames).astype(np.float64)
    nk = nq if not g.cached_t else np.concatenate([block_token_counts(g, g.cached_t), nq])
    sel = np.arange(idx.shape[-1])[None, None, None, :] < cnt[..., None]
    nj = np.where(sel, nk[np.clip(idx, 0, None)], 0.0).sum(axis=-1)  # [B, H, NBq]
    return float(4.0 * g.head_dim * (nj * nq[None, None, :]).sum())


def selection_locality(g, idx: np.ndarray, cnt: np.ndarray) -> float:
    """Share of selected key blocks within one block (t, h or w) of their query block."""
    per_t = -(-g.grid_h // g.blk[1]) * -(-g.grid_w // g.blk[2])
    nbw = -(-g.grid_w // g.blk[2])
    nbc = (g.cached_t // g.blk[0]) * per_t
    sel = np.arange(idx.shape[-1])[None, None, None, :] < cnt[..., None]
    i = np.arange(idx.shape[2])[None, None, :, None] + nbc  # global position of the query block
    j = np.clip(idx, 0, None)
    d = np.maximum(np.abs(i // per_t - j // per_t),
                   np.maximum(np.abs((i % per_t) // nbw - (j % per_t) // nbw), np.abs(i % nbw - j % nbw)))
    return float(((d <= 1) & sel).sum() / max(1, sel.sum()))


def traffic_per_launch(kernel, workload, n_pairs, n_pairs_cur):
    b = DRAM_BYTES_PER_PAIR.get(kernel)
    if b is None:
        return None
    return b * (n_pairs_cur if kernel == "bwd_dkdv" else n_pairs)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


def cpu_oracle_sample(w, budget_s: float = 12.0, with_bwd: bool = True):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload: prologue and
    routing of one head, forward attention of as many query blocks of that head as fit 40 %
    of the budget and, with the backward, the backward of as many as fit the rest.  The rate
    is the step's: tile FLOPs of one query block's forward plus 2.5x that backward, over the
    oracle's time per query block (routing prorated over the head's query blocks)."""
    import oracle
    grid = oracle.Grid(w.t_frames, w.grid_h, w.grid_w, w.blk, w.cached_t, w.chunk_t, w.cond_t)
    x = make_raster_inputs(w, with_grad=True)
    from synth import bf16_bits_to_f64
    h = 0
    q = bf16_bits_to_f64(x["q"][:, :, h:h + 1])
    k = bf16_bits_to_f64(x["k"][:, :, h:h + 1])
    v = bf16_bits_to_f64(x["v"][:, :, h:h + 1])
    do = bf16_bits_to_f64(x["do"][:, :, h:h + 1])
    kc = bf16_bits_to_f64(x["kc"][:, :, h:h + 1]) if w.cached_t else None
    vc = bf16_bits_to_f64(x["vc"][:, :, h:h + 1]) if w.cached_t else None
    gq = x["gamma_q"] if w.qknorm else None
    gk = x["gamma_k"] if w.qknorm else None
    theta = w.theta if w.rope else 0.0
    scale = 1.0 / np.sqrt(w.head_dim)
    t0 = time.perf_counter()
    qp = oracle.prologue(q, w.t_frames, w.grid_h, w.grid_w, gamma=gq, eps=w.eps, theta=theta,
                         t_offset=w.cached_t)
    kp = oracle.prologue(k, w.t_frames, w.grid_h, w.grid_w, gamma=gk, eps=w.eps, theta=theta,
                         t_offset=w.cached_t)
    idx, cnt, _ = oracle.route(qp, kp, grid, w.top_r, k_cache=kc)
    t_route = time.perf_counter() - t0
    order = np.random.default_rng(0).permutation(grid.nbq)

    def timed(fn, budget):
        n, t = 0, 0.0
        while t < budget and n < grid.nbq:
            t1 = time.perf_counter()
            fn(int(order[n]))
            t += time.perf_counter() - t1
            n += 1
        return n, t

    n_f, t_f = timed(lambda i: oracle.attend(qp, kp, v, idx, grid, scale, k_cache=kc, v_cache=vc,
                                             query_blocks=[(0, 0, i)]),
                     budget_s * (0.4 if with_bwd else 1.0))
    n_b, t_b = timed(lambda i: oracle.attend_bwd(qp, kp, v, do, idx, grid, scale, k_cache=kc,
                                                 v_cache=vc, query_blocks=[(0, 0, i)]),
                     budget_s * 0.6) if with_bwd else (0, 0.0)
    pairs = float(np.mean(cnt[0, 0]))  # selected key blocks per query block
    fl_blk = tile_flops(grid.bs, w.head_dim, 1) * pairs
    t_blk = t_f / n_f + (t_b / n_b if n_b else 0.0) + t_route / grid.nbq
    fl = fl_blk * (3.5 if with_bwd else 1.0)
    cores = len(os.sched_getaffinity(0))
    out = {
        "value": fl / t_blk / 1e12,
        "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
        "fwd_tflops": fl_blk / (t_f / n_f) / 1e12,
        "sample": f"fp64 oracle: prologue+route of 1/{w.heads} heads, forward attention of "
                  f"{n_f} query blocks of that head" +
                  (f" and backward of {n_b}" if with_bwd else "") +
                  f" ({pairs:.0f} key blocks each); rate = (fwd + 2.5x fwd) tile FLOPs per "
                  f"query block over fwd + bwd + prorated route time per query block; "
                  f"{t_f + t_b + t_route:.1f} s of CPU work",
    }
    if with_bwd:
        out["bwd_tflops"] = 2.5 * fl_blk / (t_b / n_b) / 1e12
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="720p", choices=["720p", "480p", "480p_cont"])
    ap.add_argument("--no-bwd", action="store_true", help="forward path only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--structured", action="store_true",
                    help="q and k share a smooth low-frequency field (video-like routing locality)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    with_bwd = not args.no_bwd

    if args.impl == "reference":
        if rank != 0:
            return 0
        t0 = time.perf_counter()
        vals = [cpu_oracle_sample(w, budget_s=max(2.0, 60.0 / max(1, args.steps + args.warmup)),
                                  with_bwd=not args.no_bwd)
                for _ in range(args.warmup + args.steps)][args.warmup:]
        v = float(np.median([x["value"] for x in vals]))
        cb = dict(vals[-1])
        cb["value"] = v
        line = {"impl": "reference", "metric": "BSA fwd(+bwd) effective TFLOP/s at 720p tokens",
                "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": args.workload, "tokens": w.n_tokens, "heads": w.heads,
                           "head_dim": w.head_dim, "block": list(w.blk), "top_r": w.top_r},
                "cpu_baseline": cb,
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "wall_s": time.perf_counter() - t0}
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.pipeline import BsaPipeline

    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    g = bsa.Geometry.from_workload(w)
    x = make_raster_inputs(w, with_grad=with_bwd, seed_offset=0)
    if args.structured:
        x = add_smooth_field(w, x)

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    pipe = BsaPipeline(g, w.top_r, rope_theta=w.theta if w.rope else 0.0, qknorm=w.qknorm,
                       eps=w.eps, with_bwd=with_bwd, device=str(dev))
    if w.qknorm:
        pipe.set_gamma(torch.from_numpy(x["gamma_q"]).to(dev), torch.from_numpy(x["gamma_k"]).to(dev))
    if w.cached_t:
        pipe.load_cache(dev_bf16(x["kc"]), dev_bf16(x["vc"]))
    q_d, k_d, v_d = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    if with_bwd:
        do_d = dev_bf16(x["do"])
        pipe.load_grad(do_d)
    stream = torch.cuda.current_stream(dev)

    ev = {}

    def step(record: bool):
        marks = []
        if record:
            marks.append(torch.cuda.Event(enable_timing=True)); marks[-1].record(stream)
        pipe.prologue(q_d, k_d, v_d, stream)
        if record:
            marks.append(torch.cuda.Event(enable_timing=True)); marks[-1].record(stream)
        pipe.route(stream)
        if record:
            marks.append(torch.cuda.Event(enable_timing=True)); marks[-1].record(stream)
        pipe.attn_fwd(stream)
        if record:
            marks.append(torch.cuda.Event(enable_timing=True)); marks[-1].record(stream)
        if with_bwd:
            pipe.backward(stream)
            if record:
                marks.append(torch.cuda.Event(enable_timing=True)); marks[-1].record(stream)
        return marks

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    st = bsa.bsa_device_status()
    if st != 0:
        raise SystemExit(f"device status {st} after warm-up")

    n_pairs = int(pipe.cnt.sum().item())
    r_idx = torch.arange(w.top_r, device=dev).view(1, 1, 1, -1)
    sel = r_idx < pipe.cnt.unsqueeze(-1)
    n_pairs_cur = int(((pipe.idx >= g.nbc) & sel).sum().item())  # pairs with a current key block
    fl_fwd = tile_flops(g.bs, g.head_dim, n_pairs)
    fl_step = fl_fwd * (3.5 if with_bwd else 1.0)
    idx_h, cnt_h = pipe.idx.cpu().numpy(), pipe.cnt.cpu().numpy()
    fl_fwd_valid = valid_token_flops(g, idx_h, cnt_h)
    locality = selection_locality(g, idx_h, cnt_h)

    barrier()
    torch.cuda.synchronize()
    all_marks = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    bsa.bsa_kernel_timing(True)  # event pairs around each attention kernel, on its stream
    with ClockSampler(dev.index or 0) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            all_marks.append(step(True))
        t1.record(stream)
        torch.cuda.synchronize()
    ktimes = bsa.bsa_kernel_time_stats()
    bsa.bsa_kernel_timing(False)
    barrier()
    ms = t0.elapsed_time(t1) / args.steps
    names = ["prologue", "route", "fwd"] + (["bwd"] if with_bwd else [])
    parts = {n: float(np.mean([m[i].elapsed_time(m[i + 1]) for m in all_marks]))
             for i, n in enumerate(names)}
    st = bsa.bsa_device_status()
    if st != 0:
        raise SystemExit(f"device status {st} after timing")

    ms_max = ms
    if world > 1:
        tt = torch.tensor([ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms_max = float(tt.item())

    # ---------------- end to end through the public pipeline, host buffers in and out.
    # Every step copies its raster q, k, v (and dO with the backward) in from pinned host
    # memory and its results out: O turned back to the raster layout by the inverse relayout
    # and, with the backward, the raster gradients dq, dk, dv of the step's raster inputs
    # (attention backward, then the prologue backward through RoPE and RMSNorm).  The copies
    # run on their own streams so that step k+1's upload and step k's download overlap the
    # compute (two device sets of inputs and of outputs; events order every reuse).
    in_keys = ("q", "k", "v") + (("do",) if with_bwd else ())
    out_keys = ("o",) + (("dq", "dk", "dv") if with_bwd else ())
    pin = {k_: torch.from_numpy(x[k_].view(np.int16)).pin_memory() for k_ in in_keys}
    host_out = {k_: torch.empty(q_d.shape, dtype=torch.int16).pin_memory() for k_ in out_keys}
    e_steps = max(3, args.steps)  # as many as the timed steps; the first upload is pipeline fill
    sets = [{k_: torch.empty_like(q_d) for k_ in in_keys} for _ in range(2)]
    outs = [{k_: torch.empty_like(q_d) for k_ in out_keys} for _ in range(2)]
    dgq_e = torch.empty(w.head_dim, device=dev)
    dgk_e = torch.empty(w.head_dim, device=dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]    # inputs of step k on the device
        ev_free = [torch.cuda.Event() for _ in range(n)]  # step k no longer reads its inputs
        ev_o = [torch.cuda.Event() for _ in range(n)]     # raster O of step k written
        ev_done = [torch.cuda.Event() for _ in range(n)]  # every output of step k written
        ev_out = [torch.cuda.Event() for _ in range(n)]   # outputs of step k copied out
        for k_ in range(n):
            src, dst = sets[k_ % 2], outs[k_ % 2]
            with torch.cuda.stream(up):
                if k_ >= 2:
                    up.wait_event(ev_free[k_ - 2])
                for key in in_keys:
                    src[key].view(torch.int16).copy_(pin[key], non_blocking=True)
                ev_in[k_].record(up)
            stream.wait_event(ev_in[k_])
            if k_ >= 2:
                stream.wait_event(ev_out[k_ - 2])  # this output set has been copied out
            pipe.prologue(src["q"], src["k"], src["v"], stream)
            pipe.route(stream)
            pipe.attn_fwd(stream)
            pipe.o_to_raster(dst["o"], stream)
            ev_o[k_].record(stream)
            if with_bwd:
                pipe.load_grad(src["do"], stream)
                pipe.backward(stream)
                pipe.prologue_backward(src["q"], src["k"], dst["dq"], dst["dk"], dst["dv"],
                                       dgq_e, dgk_e, stream)
            ev_free[k_].record(stream)
            ev_done[k_].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_o[k_])
                host_out["o"].copy_(dst["o"].view(torch.int16), non_blocking=True)
                down.wait_event(ev_done[k_])
                for key in out_keys[1:]:
                    host_out[key].copy_(dst[key].view(torch.int16), non_blocking=True)
                ev_out[k_].record(down)
        return ev_out[-1]

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    last = e2e_run(e_steps)
    stream.wait_event(last)
    e1.record(stream)
    torch.cuda.synchronize()
    st = bsa.bsa_device_status()
    if st != 0:
        raise SystemExit(f"device status {st} after the end-to-end run")
    e_ms = e0.elapsed_time(e1) / e_steps
    if world > 1:
        tt = torch.tensor([e_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e_ms = float(tt.item())
    h2d = sum(pin[k_].numel() * 2 for k_ in pin)
    d2h = sum(host_out[k_].numel() * 2 for k_ in host_out)
    del sets, outs

    # ---------------- the next row of the path, timed on its own (not part of the step):
    # the prologue backward, raster q, k, v gradients and the gains' gradients from the
    # attention backward's blocked dq, dk, dv
    next_rows = {}
    if with_bwd:
        pb = [torch.empty_like(q_d) for _ in range(3)]
        dgq = torch.empty(w.head_dim, device=dev)
        dgk = torch.empty(w.head_dim, device=dev)
        for _ in range(2):
            pipe.prologue_backward(q_d, k_d, pb[0], pb[1], pb[2], dgq, dgk, stream)
        torch.cuda.synchronize()
        p0 = torch.cuda.Event(enable_timing=True)
        p1 = torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        for _ in range(args.steps):
            pipe.prologue_backward(q_d, k_d, pb[0], pb[1], pb[2], dgq, dgk, stream)
        p1.record(stream)
        torch.cuda.synchronize()
        p_ms = p0.elapsed_time(p1) / args.steps
        # read blocked dq, dk, dv and raster q, k; write raster dq, dk, dv
        p_bytes = 3 * pipe.dq.numel() * 2 + 5 * q_d.numel() * 2
        next_rows["prologue_bwd"] = {"ms_per_call": p_ms, "bytes": p_bytes,
                                     "gbs": p_bytes / (p_ms * 1e-3) / 1e9}

    # the continuation cache for the next round: this geometry's blocked K, V and key-block
    # means appended to a cache of as many frames (the blocked Q, O and Q means stand in for
    # it: distinct buffers, so no source is read twice through L2)
    if w.t_frames % w.blk[0] == 0:
        gc = dataclasses.replace(g, cached_t=w.t_frames)
        cshape = (g.batch, g.heads, 2 * g.nbq, g.bs, g.head_dim)
        kc_n = torch.empty(cshape, dtype=torch.bfloat16, device=dev)
        vc_n = torch.empty_like(kc_n)
        kp_n = torch.empty(cshape[:3] + (g.head_dim,), dtype=torch.float32, device=dev)
        ca = lambda: bsa.bsa_cache_append(gc, pipe.q, pipe.o, pipe.q_pool, pipe.k, pipe.v,  # noqa: E731
                                          pipe.k_pool, kc_n, vc_n, kp_n, stream=stream)
        for _ in range(2):
            ca()
        torch.cuda.synchronize()
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(args.steps):
            ca()
        c1.record(stream)
        torch.cuda.synchronize()
        c_ms = c0.elapsed_time(c1) / args.steps
        c_bytes = 2 * (kc_n.numel() * 2 * 2 + kp_n.numel() * 4)  # read + write K, V, means
        next_rows["cache_append"] = {"ms_per_call": c_ms, "bytes": c_bytes,
                                     "gbs": c_bytes / (c_ms * 1e-3) / 1e9,
                                     "cached_t": gc.cached_t}
        del kc_n, vc_n, kp_n

    # sequence-parallel relayouts of one rank of 8 (all shards on this GPU): the sharded
    # prologue reading 8 frame shards for its 1/8 of the heads, and the inverse relayout of its
    # O into the 8 shards; bytes = its share of the raster reads / writes plus blocked outputs
    if w.t_frames % 8 == 0 and w.heads % 8 == 0 and not w.cached_t:
        from block_sparse_attention_route_b200.ulysses import UlyssesPlan
        plan = UlyssesPlan(8, 0, w.heads, w.t_frames)
        gl = plan.local_geometry(g)
        tps = plan.shard_tokens(g)
        shq, shk, shv = ([t[:, s * tps:(s + 1) * tps] for s in range(8)] for t in (q_d, k_d, v_d))
        o_ras = torch.empty_like(q_d)
        sho = [o_ras[:, s * tps:(s + 1) * tps] for s in range(8)]
        blk = [torch.empty(bsa.blocked_shape(gl), dtype=torch.bfloat16, device=dev) for _ in range(3)]
        pools = [torch.empty(bsa.blocked_shape(gl)[:3] + (g.head_dim,), dtype=torch.float32,
                             device=dev) for _ in range(2)]
        gq = pipe.gamma_q if w.qknorm else None
        gk = pipe.gamma_k if w.qknorm else None

        def u_pro():
            bsa.rope3d_qknorm_prologue_sharded(gl, w.t_frames, 0, plan.shards(), shq, shk, shv, gq,
                                               gk, w.eps, w.theta if w.rope else 0.0, blk[0],
                                               blk[1], blk[2], pools[0], pools[1], stream=stream)

        def u_out():
            bsa.bsa_blocked_to_raster_sharded(gl, w.t_frames, plan.shards(), blk[0], sho,
                                              stream=stream)
        u_rows = {}
        for nm, fn, nbytes in (("prologue", u_pro, 3 * (q_d.numel() // 8) * 2 + 3 * blk[0].numel() * 2),
                               ("o_relayout", u_out, (q_d.numel() // 8) * 2 + blk[0].numel() * 2)):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
            u_rows[nm] = {"ms_per_call": ms, "bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9}
        next_rows["ulysses_rank_of_8_local_shards"] = u_rows
        del blk, pools, o_ras, sho

    # routing variants (bsa_route_ex flags) on this workload's q / k: ms per route call
    rv = {}
    for vname, vflags in (("plain", 0), ("force_self", bsa.ROUTE_FORCE_SELF),
                          ("shared_heads", bsa.ROUTE_SHARED_HEADS),
                          ("pool_sum", bsa.ROUTE_POOL_SUM), ("pool_max", bsa.ROUTE_POOL_MAX)):
        for _ in range(2):
            pipe.route(stream, flags=vflags)
        torch.cuda.synchronize()
        r0 = torch.cuda.Event(enable_timing=True)
        r1 = torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for _ in range(args.steps):
            pipe.route(stream, flags=vflags)
        r1.record(stream)
        torch.cuda.synchronize()
        rv[vname] = r0.elapsed_time(r1) / args.steps
    pipe.route(stream)  # leave the plain selection in place
    next_rows["route_variants_ms"] = rv

    peaks = load_peaks()
    peak = peaks["bf16_tflops_sustained"]
    peak_burst = peaks["bf16_tflops"]
    # tensor FLOPs per launch of each attention kernel in 128x128xD GEMM tiles (2*BS*BS*D each).
    # Executed: forward S and PV per selected pair; dK/dV pass S^T, dP^T, dV, dK per pair with a
    # current key block; dQ pass S, dP, dQ per selected pair.  Algorithmic: the same, except that
    # the dQ pass's S and dP repeat the dK/dV pass's and are not counted (dQ = dS K only), so
    # the backward's algorithmic total is the usual 5 tiles per pair, 2.5x the forward.
    half = 0.5 * tile_flops(g.bs, g.head_dim, 1)  # one GEMM tile
    kflops = {"fwd": 2 * half * n_pairs, "bwd_dkdv": 4 * half * n_pairs_cur,
              "bwd_dq": 3 * half * n_pairs}
    kflops_alg = {"fwd": 2 * half * n_pairs, "bwd_dkdv": 4 * half * n_pairs_cur,
                  "bwd_dq": 1 * half * n_pairs}
    kernels = {}
    for kname, (nl, tot_ms, min_ms, med_ms) in ktimes.items():
        if nl == 0:
            continue
        avg = tot_ms / nl
        kernels[kname] = {"launches": nl, "ms_per_launch": avg, "ms_median": med_ms,
                          "ms_min": min_ms,
                          "tflops_executed": kflops[kname] / (avg * 1e-3) / 1e12,
                          "tflops_algorithmic": kflops_alg[kname] / (avg * 1e-3) / 1e12}
        kernels[kname]["frac_algorithmic"] = kernels[kname]["tflops_algorithmic"] / peak
    dom = max(kernels, key=lambda k_: kernels[k_]["ms_per_launch"])
    achieved = kernels[dom]["tflops_algorithmic"]
    value = world * fl_step / (ms_max * 1e-3) / 1e12
    fwd_ms, bwd_ms = parts["fwd"], parts.get("bwd")
    line = {
        "metric": "BSA fwd(+bwd) effective TFLOP/s at 720p tokens",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic, q/k with a shared smooth field" if args.structured else "synthetic",
        "config": {"workload": args.workload, "tokens": w.n_tokens, "padded_tokens": g.nbq * g.bs,
                   "heads": w.heads, "head_dim": w.head_dim, "block": list(w.blk),
                   "top_r": w.top_r, "selected_pairs": n_pairs, "with_bwd": with_bwd,
                   "fwd_tflop_tiles": fl_fwd / 1e12, "fwd_tflop_valid_tokens": fl_fwd_valid / 1e12,
                   "selections_within_one_block": locality,
                   "parallelism": f"replicas{world}", "l2": "inputs larger than L2 (126 MB)"},
        "ms_per_call": parts,
        "kernels": kernels,
        "roofline": {"bound": "tensor", "kernel": KERNEL_NAMES[dom], "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "frac_burst": achieved / peak_burst, "peak_burst": peak_burst,
                     "peak_source": f"{peaks['source']} bf16 dense, sustained (of measured)"
                                    if peaks["source"] == "measured" else "fallback",
                     "traffic": traffic_per_launch(dom, args.workload, n_pairs, n_pairs_cur),
                     "fwd_frac": fl_fwd / (fwd_ms * 1e-3) / 1e12 / peak,
                     "bwd_algorithmic_frac": (2.5 * fl_fwd / (bwd_ms * 1e-3) / 1e12 / peak
                                              if with_bwd else None),
                     "step_frac": value / world / peak, "step_frac_burst": value / world / peak_burst,
                     "note": "achieved = algorithmic GEMM-tile FLOPs of the kernel / its mean "
                             "launch time; fwd_frac, bwd_algorithmic_frac and step_frac use the "
                             "step's phase times (forward 2 tiles per pair, backward 5, step 7)"},
        "e2e": {"value": world * fl_step / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "copied_in": list(in_keys), "copied_out": [k_ + "_raster" for k_ in out_keys],
                "path": "prologue, route, fwd, O to raster" +
                        (", dO relayout, bwd, prologue bwd" if with_bwd else "")},
        "next_rows": next_rows,
        "gpu_launches": args.steps * (3 + (4 if with_bwd else 0)),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(w, with_bwd=with_bwd)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
