#!/usr/bin/env python
"""Benchmark of the FlashLoop lazy loop-r attention sublayer on B200.

One step = loops 2..R (gate, gathered QKV + RoPE, residual quantisation,
column selection, selected-column reconstruction, sparse attention update,
gathered output projection) of one synthetic 32K-token sequence per GPU,
from the untouched loop-1 state.  The metric is tokens/s = S * (R - 1) per
sequence per step, summed over ranks (weak scaling: each rank owns its own
sequence; there is no exchange between ranks).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workload import CONFIGS, make_decode_tokens, make_hidden_states, make_weights  # noqa: E402

METRIC = "loop-step tokens/s at S=32K,R=4; HBM GB/s and tensor-pipe % of B200 peak"
DECODE_METRIC = "decode tokens/s (B sequences x 1 token x R loops) at S_ctx=32K,R=4; HBM GB/s of B200 peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one launch of the dominant kernel, from the ncu captures summarised
# under profiles/; None once the kernel changes until it is re-captured.
ATTN_LOOP2_TRAFFIC = {"attn_pp_kernel<128>": 479589376 + 271851776}
ATTN_KERNEL = "attn_pp_kernel<128>"
# captured on 2 sequences and scaled by 4 (traffic in proportion to the columns read)
DECODE_DENSE_TRAFFIC = {"decode_dense_kernel<128,8>": 1169.5e6}
L2_BYTES = 126e6  # B200 L2 (126 MB)


def max_over_ranks(value, device=None):
    """Largest value over all ranks (identity on a single process)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def run_config(cfg, world, active_tokens, pairs):
    """The config object of both arms' lines (identical keys and values for
    the same workload, so the two lines compare)."""
    x_mib = cfg.seq * cfg.d_model * 2 / 2**20            # one bf16 X_r
    n_mib = cfg.n_heads * cfg.seq * cfg.head_dim * 4 / 2**20  # one float32 N slot
    size = "larger" if cfg.seq * cfg.d_model * 2 > L2_BYTES else "smaller"
    return {"workload": workload_desc(cfg),
            "l2": f"inputs {size} than L2 (126 MB): each X_r is {x_mib:g} MiB and the N state "
                  f"{n_mib:g} MiB per slot",
            "parallelism": f"one sequence per rank, {world} rank(s), no exchange",
            "active_tokens": {f"loop{r}": int(n) for r, n in sorted(active_tokens.items())},
            "attention_pairs": {f"loop{r}": int(v) for r, v in sorted(pairs.items())}}


def workload_desc(cfg):
    return (f"{cfg.name}: d_model {cfg.d_model}, {cfg.n_heads} heads x {cfg.head_dim}, S {cfg.seq}, "
            f"R {cfg.n_loops}, tau {cfg.tau}, top-k {cfg.k}/head, active "
            f"{'/'.join(f'{int(f * 100)}%' for f in cfg.active_fracs)}, bits "
            f"{'/'.join(str(b) for b in cfg.bits)}")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # the sampler takes a moment to start: wait for its first line so
        # that the samples fall inside the timed region that follows
        t_end = time.time() + 3.0
        while time.time() < t_end and os.path.getsize(self.path) == 0:
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [t.strip() for t in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


# ----------------------------------------------------------------------------- CUDA arm
def attention_pairs(active, cols):
    """Causal-valid (i, j, h) pairs: i active, j selected for head h, j <= i."""
    return int(sum(np.searchsorted(c, active, side="right").sum() for c in cols))


def run_cuda(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from cross_loop_sparse_b200 import flashloop as F

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg, b=rank)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    xs = [to_dev(x) for x in X]
    wqkv, wo = to_dev(W["wqkv"]), to_dev(W["wo"])
    paper = args.kv_scheme == "paper"
    p = F.Params.from_config(cfg, fixed_mass=args.fixed_mass, kv_scheme=args.kv_scheme)
    st = F.FlashLoopState(p, device=dev)
    S, d, R = cfg.seq, cfg.d_model, cfg.n_loops
    F.flashloop_loop_step(p, 1, xs[0], None, wqkv, wo, st)
    torch.cuda.synchronize()
    if paper:
        kf = torch.empty((S, d), dtype=torch.float32, device=dev)
        vf = torch.empty_like(kf)

    def project_quant(r, x, act, n_act, cap, q_out):
        """Projection of the loop's active rows with its K/V quantisation:
        fused into the GEMM epilogue (INT8 + INT4/INT2 streams), or the
        gathered projection then the asymmetric INT4 quantiser (the pages'
        setting).  Returns the launches made."""
        if not paper:
            F.flashloop_qkv_quant(p, r, x, act, n_act, wqkv, st, q_out)
            return 1
        F.flashloop_qkv_gathered(p, x, act, n_act, cap, wqkv, st["rope_cs"], q_out, kf, vf)
        F.flashloop_paper_kv_quant(p, r, kf, vf, act, n_act, st)
        return 4

    # Loop 1 (the dense producer of the base cache, the state and the column
    # mass), timed on its own: it runs once per sequence, before the loop steps.
    # Re-running it rewrites slot 0 with the same bytes.
    def loop1(events):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        ev[0].record(stream)
        project_quant(1, xs[0], None, None, S, st["q0"])
        ev[1].record(stream)
        F.flashloop_selcol_dequant(p, 1, st)
        ev[2].record(stream)
        F.flashloop_sparse_attn_update(p, 1, st, 1)
        ev[3].record(stream)
        F.flashloop_out_proj(p, st["O"], None, None, S, wo, st["Y"])
        ev[4].record(stream)
        events.append(ev)

    l1_events = []
    for i in range(4):
        loop1(l1_events if i > 0 else [])
    torch.cuda.synchronize()
    l1 = {k: statistics.mean(e[a].elapsed_time(e[b]) for e in l1_events)
          for k, a, b in (("ms", 0, 4), ("qkv_quant", 0, 1), ("rebuild", 1, 2), ("attention_colmass", 2, 3),
                          ("out_proj", 3, 4))}

    launches_per_step = 0
    attn_events = []

    def step(record):
        nonlocal launches_per_step
        n = 0
        for r in range(2, R + 1):
            act, n_act = st[f"active{r}"], st["n_active"][r - 1:]
            prev = None if r == 2 else st[f"active{r - 1}"]
            n_prev = None if r == 2 else st["n_active"][r - 2:]
            F.flashloop_gate(p, xs[r - 1], xs[r - 2], prev, n_prev, p.capacity[r - 2] if r > 2 else S,
                             act, st[f"slot{r}"], n_act, p.capacity[r - 1], st["workspace"], st["err"])
            n += 1 + project_quant(r, xs[r - 1], act, n_act, p.capacity[r - 1], st[f"q{st.q_slot(r)}"])
            if F.flashloop_selection_loop(p, r) == r:
                src = st["colmass0"] if r == 2 else st["colmass1"]
                F.flashloop_topk_columns(p, src, None, 0, p.topk[r - 1], st[f"cols{r}"])
                n += 1
            F.flashloop_selcol_dequant(p, r, st)
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            F.flashloop_sparse_attn_update(p, r, st, 0)
            if record:
                e1.record(stream)
                attn_events.append((r, e0, e1))
            F.flashloop_out_proj(p, st["O"], act, n_act, p.capacity[r - 1], wo, st["Y"])
            n += 4 if p.fixed_mass else 3  # the fixed-mass form runs a statistics and an update pass
        launches_per_step = n

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    barrier()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local_rank)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        step(True)
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    err = st.error_code()
    if err != 0:
        raise RuntimeError(f"device error word {err}")

    # Algorithmic work of the dominant kernel (attention update): 8*dh FLOP
    # per causal-valid (active row, selected column, head) pair.
    pairs = {}
    for r in range(2, R + 1):
        n = int(st["n_active"][r - 1].item())
        act = st[f"active{r}"][:n].cpu().numpy()
        cols = st.cols_for_loop(r).cpu().numpy()
        pairs[r] = attention_pairs(act, cols)
    per_loop = {}
    for r, e0, e1 in attn_events:
        per_loop.setdefault(r, []).append(e0.elapsed_time(e1))
    attn_ms = sum(sum(v) for v in per_loop.values())
    peaks, peak_kind = load_peaks()
    # The dominant kernel is the attention update; its largest launch (loop 2) is the one reported.
    ms2 = statistics.mean(per_loop[2])
    flop2 = 8 * cfg.head_dim * pairs[2]
    achieved = flop2 / (ms2 * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": None if args.fixed_mass else ATTN_LOOP2_TRAFFIC.get(ATTN_KERNEL),
                "kernel": ("attn_tc_kernel<128> statistics + update passes, loop 2 (fixed-mass form, tcgen05)"
                           if args.fixed_mass else
                           f"{ATTN_KERNEL}, loop-2 launch (sparse attention update, tcgen05)"),
                "algorithmic": f"8*dh FLOP x {pairs[2]} causal-valid (row, column, head) pairs = {flop2:.4g} FLOP",
                "peak_source": f"{peak_kind} bf16 dense burst (fp16 operands run at the bf16 rate)",
                "per_loop": {f"loop{r}": {"ms": round(statistics.mean(v), 4),
                                          "tflops": round(8 * cfg.head_dim * pairs[r] / (statistics.mean(v) * 1e-3) / 1e12, 2)}
                             for r, v in sorted(per_loop.items())},
                "attn_share_of_step": round(attn_ms / ms, 4)}

    # End to end through the public API with host buffers, pipelined the way a
    # serving loop runs it: every step copies its hidden states X_2..X_R from
    # pinned host memory on a copy stream into one of two device buffer sets
    # (the next step's copies overlap this step's compute), loop_step r waits
    # for X_r only, and Y goes back to the host on a second copy stream once
    # loop R is done.  Y alternates between two device buffers (the second
    # starts as a copy of the first, so rows a step leaves untouched agree)
    # so that the next step need not wait for the read-back.
    host_x = [torch.from_numpy(X[r - 1].view(np.int16)).view(torch.bfloat16).pin_memory()
              for r in range(2, R + 1)]
    host_y = torch.empty((S, d), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(2, min(args.steps, 10))
    xbuf = [[torch.empty_like(xs[r - 1]) for r in range(2, R + 1)] for _ in range(2)]
    ybuf = [st["Y"], st["Y"].clone()]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    set_free = [None, None]  # the last compute that read each X buffer set
    y_free = [None, None]    # the last read-back of each Y buffer

    def e2e_step(sidx):
        b = sidx % 2
        ready = []
        if set_free[b] is not None:
            h2d.wait_event(set_free[b])
        with torch.cuda.stream(h2d):
            for i in range(R - 1):
                xbuf[b][i].copy_(host_x[i], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(h2d)
                ready.append(ev)
        if y_free[b] is not None:
            stream.wait_event(y_free[b])
        st.c.Y = ybuf[b].data_ptr()
        for i, r in enumerate(range(2, R + 1)):
            stream.wait_event(ready[i])
            x_prev = xs[0] if r == 2 else xbuf[b][i - 1]
            F.flashloop_loop_step(p, r, xbuf[b][i], x_prev, wqkv, wo, st, stream)
        done = torch.cuda.Event()
        done.record(stream)
        set_free[b] = done
        d2h.wait_event(done)
        with torch.cuda.stream(d2h):
            host_y.copy_(ybuf[b], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(d2h)
        y_free[b] = ev

    e2e_step(0)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i + 1)
    for ev in y_free:
        stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize()
    st.c.Y = ybuf[0].data_ptr()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    barrier()

    tokens = S * (R - 1) * world
    ms_step = ms / args.steps
    # Whole step against the tensor roofline: attention 8*dh FLOP per causal-valid
    # pair plus the gathered projections 8*d^2 FLOP per active row (QKV 6, W_o 2).
    n_act = {r: int(st["n_active"][r - 1].item()) for r in range(2, R + 1)}
    attn_flop = sum(8 * cfg.head_dim * pairs[r] for r in range(2, R + 1))
    gemm_flop = sum(8 * d * d * n_act[r] for r in range(2, R + 1))
    step_tflops = (attn_flop + gemm_flop) / (ms / args.steps * 1e-3) / 1e12
    step_roofline = {"bound": "tensor", "flop": int(attn_flop + gemm_flop), "attention_flop": int(attn_flop),
                     "projection_flop": int(gemm_flop), "achieved": round(step_tflops, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(step_tflops / peaks["bf16_tflops"], 4),
                     "roofline_ms": round((attn_flop + gemm_flop) / (peaks["bf16_tflops"] * 1e12) * 1e3, 4)}
    # loop 1: projections 8*d^2 per token, dense causal attention 4*dh per pair and
    # head, the column mass's score recomputation 2*dh per pair and head
    pairs1 = S * (S + 1) // 2 * cfg.n_heads
    l1_flop = 8 * d * d * S + 6 * cfg.head_dim * pairs1
    loop1_line = {"ms": round(l1["ms"], 4), "tokens_per_s": round(S / (l1["ms"] * 1e-3), 1),
                  "kernels_ms": {k: round(v, 4) for k, v in l1.items() if k != "ms"},
                  "flop": int(l1_flop), "achieved": round(l1_flop / (l1["ms"] * 1e-3) / 1e12, 2),
                  "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                  "frac": round(l1_flop / (l1["ms"] * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                  "roofline_ms": round(l1_flop / (peaks["bf16_tflops"] * 1e12) * 1e3, 4)}
    variants = []
    # a variant of the path: the config says so (the reference arm has no such line)
    if args.fixed_mass:
        variants.append("fixed-mass form of the update")
    if paper:
        variants.append("the pages' cache setting (INT4 asymmetric groups of 64, 64-token bf16 tail)")
    variant = ", ".join(variants) or None
    out = {
        "metric": METRIC, "value": round(tokens / (ms_step * 1e-3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded workload generator; random-init weights of the stated shape)",
        "config": run_config(cfg, world, {r: int(st['n_active'][r - 1].item()) for r in range(2, R + 1)}, pairs),
        "roofline": roofline,
        "step_roofline": step_roofline,
        "loop1": loop1_line,
        "e2e": {"value": round(tokens / (e2e_ms / e2e_steps * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": (R - 1) * S * d * 2, "d2h_bytes_per_step": S * d * 2,
                "steps": e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if variant:
        out["config"]["workload"] += ", " + variant
    out["config"]["kv_cache_bytes"] = kv_cache_bytes(cfg, st, paper)
    return out


def kv_cache_bytes(cfg, st, paper):
    """Bytes of the K and V streams after loops 1..R (codes, fp16 scales and
    minima, bf16 tail values), from the active lists."""
    S, H, dh, R = cfg.seq, cfg.n_heads, cfg.head_dim, cfg.n_loops
    E = H * dh
    n = [S] + [int(st["n_active"][r - 1].item()) for r in range(2, R + 1)]
    if not paper:   # INT8 base, INT4 / INT2 residuals, an fp16 scale per group of 32
        return int(sum(2 * (nr * E * cfg.bits[i] // 8 + nr * E // 32 * 2) for i, nr in enumerate(n)))
    tail = min(64, S)
    body = S - tail
    total = 0
    for r, nr in enumerate(n, start=1):
        nb = body if r == 1 else int((st[f"active{r}"][:nr] < body).sum().item())
        nt = nr - nb
        groups_v = nb * E // 64
        groups_k = (nb + 63) // 64 * E
        total += 2 * (nb * E // 2) + 4 * (groups_v + groups_k) + 2 * nt * E * 2
    return int(total)


# ----------------------------------------------------------------------------- decode (CUDA arm)
def decode_stream_bytes(cfg, n_cols, loop, per_col_present=None):
    """Bytes of K and V codes + fp16 scales of n_cols (column, head) entries:
    the base and, for every loop 2..loop, the residual where present
    (per_col_present[l] = fraction of the columns present at loop l)."""
    dh = cfg.head_dim
    per = dh + 2 * (dh // 32)
    for l in range(2, loop + 1):
        frac = 1.0 if per_col_present is None else per_col_present[l]
        per += frac * (dh * cfg.bits[l - 1] // 8 + 2 * (dh // 32))
    return 2 * n_cols * per


def run_decode_cuda(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from cross_loop_sparse_b200 import flashloop as F

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    B, S, d, R, H, dh = cfg.batch, cfg.seq, cfg.d_model, cfg.n_loops, cfg.n_heads, cfg.head_dim
    W = make_weights(cfg)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    wqkv, wo = to_dev(W["wqkv"]), to_dev(W["wo"])
    p = F.Params.from_config(cfg)
    ctx = F.DecodeContext(p, device=dev)
    ds = F.DecodeState(p, device=dev)
    seqs = [rank * B + i for i in range(B)]
    # the contexts' caches (what their prefill leaves), built loop by loop on the GPU; untimed
    ctx_x = [make_hidden_states(cfg, b)[0] for b in seqs]
    xs = [to_dev(np.concatenate([c[r] for c in ctx_x], axis=0)) for r in range(R)]
    del ctx_x
    ctx.prepare(xs, wqkv)
    del xs
    toks = [make_decode_tokens(cfg, b) for b in seqs]
    host_tok = [np.stack([t[r] for t in toks]) for r in range(R)]
    xt = [to_dev(x) for x in host_tok]
    torch.cuda.synchronize()

    events = []

    def step(record):
        for r in range(1, R + 1):
            F.flashloop_decode_qkv(p, r, xt[r - 1], wqkv, ds)
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            F.flashloop_decode_attn(p, r, ctx, ds)
            if record:
                e1.record(stream)
                events.append((r, e0, e1))
            if r == 1:
                F.flashloop_decode_select(p, ds)
            F.flashloop_decode_out(p, wo, ds)
        # per loop: GEMV + token quantisation, attention + merge, out GEMV; top-k at loop 1
        return 5 * R + 1

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        launches = step(False)
    torch.cuda.synchronize()
    barrier()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local_rank)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        launches = step(True)
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    for name, err in (("context", ctx.error_code()), ("decode", ds.error_code())):
        if err != 0:
            raise RuntimeError(f"{name} device error word {err}")

    per_loop = {}
    for r, e0, e1 in events:
        per_loop.setdefault(r, []).append(e0.elapsed_time(e1))
    peaks, peak_kind = load_peaks()
    # loop 1 (the dominant pass): the INT8 base codes + scales of K and V of
    # every column 0..S of every (sequence, head)
    P1 = S + 1
    bytes1 = decode_stream_bytes(cfg, B * H * P1, 1)
    ms1 = statistics.mean(per_loop[1])
    achieved = bytes1 / (ms1 * 1e-3) / 1e9
    n_ctx = ctx["n_active"].cpu().numpy()
    cols = ds["cols"].cpu().numpy()
    # fraction of the selected (sequence, head, column) entries with a loop-l residual
    is_tok = cols == S
    rows = np.arange(B)[:, None, None] * S + np.minimum(cols, S - 1)
    present = {l: float(((ctx[f"slot{l}"].cpu().numpy()[rows] >= 0) | is_tok).mean()) for l in range(2, R + 1)}
    sparse = {}
    for r in range(2, R + 1):
        b_r = decode_stream_bytes(cfg, cols.size, r, present)
        m_r = statistics.mean(per_loop[r])
        sparse[f"loop{r}"] = {"ms": round(m_r, 4), "gbs": round(b_r / (m_r * 1e-3) / 1e9, 1),
                              "bytes": int(b_r)}
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": (DECODE_DENSE_TRAFFIC.get(f"decode_dense_kernel<{dh},{H * dh // 256}>")
                            if (B, S, H, dh) == (8, 32768, 16, 128) else None),
                "kernel": f"decode_dense_kernel<{dh},{H * dh // 256}> + decode_dense_merge_kernel "
                          "(loop-1 pass, timed together)",
                "algorithmic": f"K and V INT8 base codes + fp16 scales of {B}x{H}x{P1} (sequence, head, column) "
                               f"entries = {bytes1:.4g} B",
                "peak_source": f"{peak_kind} HBM copy bandwidth",
                "per_loop": {"loop1": {"ms": round(ms1, 4), "gbs": round(achieved, 1)}, **sparse},
                "attn_share_of_step": round(sum(sum(v) for v in per_loop.values()) / ms, 4)}

    # End to end through the public API with host buffers: H2D of the B tokens'
    # hidden states of loops 1..R from pinned memory, decode_step per loop,
    # D2H of Y.
    host_x = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in host_tok]
    host_y = torch.empty((B, d), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 20))

    def e2e_step():
        for r in range(R):
            xt[r].copy_(host_x[r], non_blocking=True)
        for r in range(1, R + 1):
            F.flashloop_decode_step(p, r, xt[r - 1], wqkv, wo, ctx, ds)
        host_y.copy_(ds["Y"], non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    barrier()

    tokens = B * world
    ms_step = ms / args.steps
    return {
        "metric": DECODE_METRIC, "value": round(tokens / (ms_step * 1e-3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded workload generator; random-init weights of the stated shape)",
        "config": {"workload": f"{cfg.name}: {B} sequences x 1 token at position {S} against {S}-token "
                               f"contexts, d_model {d}, {H} heads x {dh}, R {R}, top-k {cfg.k}/head, bits "
                               f"{'/'.join(str(b) for b in cfg.bits)}",
                   "l2": "inputs larger than L2: the loop-1 pass reads 1.14 GB of cache per step",
                   "parallelism": f"{B} sequences per GPU, {world} GPU(s), no exchange",
                   "context_active_rows": {f"loop{r}": int(n_ctx[r - 1]) for r in range(2, R + 1)}},
        "roofline": roofline,
        "e2e": {"value": round(tokens / (e2e_ms / e2e_steps * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": R * B * d * 2, "d2h_bytes_per_step": B * d * 2, "steps": e2e_steps},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }


class DecodeOracleSample:
    """The CPU oracle's decode on a bounded sample: one sequence, one head,
    its context part (what the prefill leaves) computed once untimed; each
    step re-runs the token's loops 1..R.  A full step is that time x B x H."""

    def __init__(self, cfg, heads=(0,)):
        import oracle as O
        self.O, self.cfg, self.heads = O, cfg, list(heads)
        self.W = make_weights(cfg)
        self.ctx = make_hidden_states(cfg, 0)[0]
        self.tok = make_decode_tokens(cfg, 0)
        self.base = O.OracleDecode(cfg, self.W, self.ctx, self.tok, heads=self.heads).prepare_context()

    def step(self):
        import copy
        orc = copy.deepcopy(self.base)
        t = time.perf_counter()
        orc.run()
        dt = time.perf_counter() - t
        scale = self.cfg.batch * self.cfg.n_heads / len(self.heads)
        sample = (f"oracle decode loops 1..{self.cfg.n_loops} of one token against a {self.cfg.seq}-token "
                  f"context on {len(self.heads)} of {self.cfg.n_heads} heads ({dt:.2f} s, includes the "
                  f"cache writes of the context rows), scaled x{scale:g} to {self.cfg.batch} sequences x "
                  f"{self.cfg.n_heads} heads")
        return dt * scale, sample


# ----------------------------------------------------------------------------- oracle timing
class OracleSample:
    """The CPU oracle on a bounded sample of the workload: loops 2..R for the
    given heads of one sequence, from a loop-1 state computed once (untimed).
    A full step is extrapolated as the gate once, the per-head work times
    H / len(heads), and the output projection from a 1024-row sample."""

    def __init__(self, cfg, heads=(0,)):
        import oracle as O
        self.O = O
        self.cfg, self.heads = cfg, list(heads)
        self.W = make_weights(cfg)
        self.X, _ = make_hidden_states(cfg)
        self.base = O.OracleSequence(cfg, self.W, self.X, heads=self.heads, keep_history=False)
        self.base.run_loop1()

    def step(self):
        import copy
        O, cfg, X = self.O, self.cfg, self.X
        orc = copy.deepcopy(self.base)
        t_gate = t_loops = t_wo = 0.0
        for r in range(2, cfg.n_loops + 1):
            t = time.perf_counter()
            O.gate(X[r - 1], X[r - 2], orc.active[r - 1], cfg.tau)
            t_gate += time.perf_counter() - t
            t = time.perf_counter()
            orc.run_loop(r)
            t_loops += time.perf_counter() - t
            n = orc.active[r].size
            rows = min(1024, n)
            t = time.perf_counter()
            O.out_projection(np.zeros((rows, cfg.d_model), np.uint16), self.W["wo"])
            t_wo += (time.perf_counter() - t) * n / rows
        t_head = max(t_loops - t_gate, 0.0)
        t_est = t_gate + t_head * cfg.n_heads / len(self.heads) + t_wo
        sample = (f"oracle loops 2..{cfg.n_loops} on {len(self.heads)} of {cfg.n_heads} heads of one "
                  f"{cfg.seq}-token sequence: gate {t_gate:.2f} s (counted once), per-head work "
                  f"{t_head:.2f} s (scaled x{cfg.n_heads / len(self.heads):g}), W_o from a 1024-row sample "
                  f"{t_wo:.2f} s (scaled to the active rows)")
        return t_est, sample

    @staticmethod
    def cores():
        try:
            from threadpoolctl import threadpool_info
            n = sum(i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas")
            return n or os.cpu_count()
        except Exception:
            return os.cpu_count()


class OracleFullStep:
    """The CPU oracle over the whole workload: loops 2..R of one sequence on
    every head, gate and output projection included, from a loop-1 state
    computed once (untimed set-up)."""

    def __init__(self, cfg):
        import oracle as O
        self.O, self.cfg = O, cfg
        self.W = make_weights(cfg)
        self.X, _ = make_hidden_states(cfg)
        t = time.perf_counter()
        self.base = O.OracleSequence(cfg, self.W, self.X, keep_history=False)
        self.base.run_loop1()
        self.setup_s = time.perf_counter() - t

    def step(self):
        import copy
        orc = copy.deepcopy(self.base)
        t = time.perf_counter()
        for r in range(2, self.cfg.n_loops + 1):
            orc.run_loop(r)
        dt = time.perf_counter() - t
        pairs = {r: attention_pairs(orc.active[r], orc.T[r]) for r in range(2, self.cfg.n_loops + 1)}
        active = {r: orc.active[r].size for r in range(2, self.cfg.n_loops + 1)}
        return dt, active, pairs


def run_reference(args, cfg):
    """The reference arm: the CPU oracle as it stands.  Prefill: one full
    step (every head), timed once; decode: a bounded sample per step."""
    if cfg.decode:
        smp = DecodeOracleSample(cfg)
        times, sample = [], ""
        for i in range(args.warmup + args.steps):
            t_est, sample = smp.step()
            if i >= args.warmup:
                times.append(t_est)
        ms = statistics.mean(times) * 1e3
        val = cfg.batch / (ms * 1e-3)
        return {
            "impl": "reference", "metric": DECODE_METRIC, "value": round(val, 4), "unit": "tokens/s",
            "n_gpus": 1, "steps": len(times), "warmup": args.warmup, "ms_per_step": round(ms, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.description, "parallelism": "CPU oracle, host cores"},
            "cpu_baseline": {"value": round(val, 4), "unit": "tokens/s", "cores": OracleSample.cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(val, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
    # A full step of the oracle takes about a minute on 16 cores (and its
    # loop-1 set-up a few), so it is timed once, with no warm-up: the line
    # reports the steps it timed, not the ones requested.
    full = OracleFullStep(cfg)
    dt, active, pairs = full.step()
    ms = dt * 1e3
    tokens = cfg.seq * (cfg.n_loops - 1)
    val = tokens / dt
    sample = (f"one full step: oracle loops 2..{cfg.n_loops} of one {cfg.seq}-token sequence on all "
              f"{cfg.n_heads} heads (gate, projections, quantisation, selection, attention, W_o), "
              f"{dt:.1f} s; loop-1 set-up {full.setup_s:.1f} s untimed")
    return {
        "impl": "reference", "metric": METRIC, "value": round(val, 2), "unit": "tokens/s", "n_gpus": 1,
        "steps": 1, "warmup": 0, "requested": {"steps": args.steps, "warmup": args.warmup},
        "ms_per_step": round(ms, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(cfg, 1, active, pairs),
        "cpu_baseline": {"value": round(val, 2), "unit": "tokens/s", "cores": OracleSample.cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(val, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--config", default="prefill_32k", choices=list(CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fixed-mass", action="store_true",
                    help="prefill workloads: the fixed-mass form of the sparse update (no CPU baseline: its "
                         "oracle keeps explicit S x S distributions)")
    ap.add_argument("--kv-scheme", choices=["spec", "paper"], default="spec",
                    help="prefill workloads: K/V streams as INT8 + INT4/INT2 symmetric residuals (spec) or the "
                         "pages' own setting, INT4 asymmetric groups of 64 with a 64-token bf16 tail (paper)")
    ap.add_argument("--batch", type=int, default=None,
                    help="decode workloads: sequences per GPU (a smaller case for profiler captures)")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]
    if args.batch is not None:
        if not cfg.decode:
            ap.error("--batch applies to decode workloads only")
        cfg = cfg.with_(batch=args.batch)
    if args.fixed_mass and (cfg.decode or args.impl != "cuda"):
        ap.error("--fixed-mass applies to the CUDA arm on prefill workloads only")
    if args.kv_scheme == "paper" and (cfg.decode or args.impl != "cuda" or args.fixed_mass):
        ap.error("--kv-scheme paper applies to the CUDA arm's running update on prefill workloads only")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    out = (run_decode_cuda if cfg.decode else run_cuda)(args, cfg, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.fixed_mass and args.kv_scheme == "spec":
        if cfg.decode:
            t_est, sample = DecodeOracleSample(cfg).step()
            value = round(cfg.batch / t_est, 4)
        else:
            t_est, sample = OracleSample(cfg).step()
            value = round(cfg.seq * (cfg.n_loops - 1) / t_est, 2)
        out["cpu_baseline"] = {"value": value, "unit": "tokens/s", "cores": OracleSample.cores(),
                               "kind": "oracle", "sample": sample}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
