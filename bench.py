#!/usr/bin/env python
"""Throughput of the block-sparse attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c4] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic inputs
already resident in HBM: block pooling of q and k (one launch), block scores +
top-k selection (two launches) and sparse attention (one launch), through the
C-ABI entry points, with CUDA events around the selection stage and the
attention on the launching stream.
value = query tokens processed by all ranks / (max over ranks of the device
time of the K timed steps). With --gpus N > 1 (under torchrun) every rank runs
its own copy of the workload on its own GPU (the (b, h) problems are
independent, so there is no data-path collective): weak scaling.

--impl reference times the float64 CPU oracle on the host cores instead (a
bounded sample of query blocks per step; rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "block-sparse attn fwd tokens/s & effective TFLOP/s (% roofline), 1 B200"

# DRAM read + write bytes per launch of the attention kernel from an ncu
# capture of the kernel as it stands, per workload; null where there is none
# (a capture of an earlier version of the kernel does not count).
NCU_TRAFFIC = {"c4": 5035535360 + 589144320}  # one launch, the current kernel
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

def max_over_ranks(x: float, dist, device) -> float:
    """The largest value of x over all ranks (the job's time is its slowest
    rank's); x itself without a process group."""
    if dist is None:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


def attn_flops(B: int, H: int, Hk: int, N: int, D: int, bs: int, kk: int, idx=None, causal: bool = False) -> float:
    """FLOPs of the attention over the kept blocks: 4 D per visible (query
    token, key token) pair (two products). Without the causal mask every
    query token sees k * bs keys: 4 B H N k bs D. With it, counted on the
    index lists `idx` ([B, H_kv, nb, k], -1 padded) the step produced: bs^2
    pairs per kept block below the query block, bs (bs + 1) / 2 for the
    diagonal block; each key/value head's lists serve H / H_kv query heads."""
    if not causal:
        return 4.0 * B * H * N * kk * bs * D
    il = np.asarray(idx, dtype=np.int64)
    qi = np.arange(N // bs)[None, None, :, None]
    pairs = np.where(il < 0, 0, np.where(il < qi, bs * bs, bs * (bs + 1) // 2)).sum()
    return 4.0 * D * float(pairs) * (H // Hk)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            pr = torch.cuda.get_device_properties(device)
            self.bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        except Exception:
            self.bus = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus:
            cmd += ["-i", self.bus]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[4], f[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[4]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------- oracle (CPU) timing

def oracle_sample(q, k, v, cfg: W.Config, heads, blocks_per_head: int, seed: int, causal=False,
                  force_diag=False):
    """Runs the oracle's whole path for `blocks_per_head` random query blocks of
    each key/value head in `heads` (each an independent problem: one head, or
    with grouped queries one key/value head and its G query heads) and returns
    (query tokens, seconds, threads)."""
    import oracle

    oracle.build()
    rng = np.random.default_rng(seed)
    G = cfg.H // cfg.Hkv
    tokens, secs = 0, 0.0
    for g in heads:
        qa = np.ascontiguousarray(W.to_oracle_array(q[:, :, g * G:(g + 1) * G]))
        ka, va = (np.ascontiguousarray(W.to_oracle_array(x[:, :, g:g + 1])) for x in (k, v))
        rows = np.sort(rng.choice(cfg.nb, size=(1, 1, blocks_per_head), replace=False), axis=-1).astype(np.int32)
        t0 = time.perf_counter()
        if G == 1:
            oracle.forward(qa, ka, va, cfg.block_size, cfg.topk_ratio, rows=rows, causal=causal,
                           force_diag=force_diag)
        else:
            oracle.forward_gqa(qa, ka, va, cfg.block_size, cfg.topk_ratio, rows=rows, causal=causal,
                               force_diag=force_diag)
        secs += time.perf_counter() - t0
        tokens += blocks_per_head * cfg.block_size * cfg.B * G
    return tokens, secs, oracle.num_threads()


def workload_config(cfg: W.Config, args, world: int, training: bool = False) -> dict:
    """The `config` object of the JSON line, the same for both arms."""
    variant = (" causal" + (" force_diag" if args.force_diag else "")) if args.causal else ""
    what = " training step (forward with lse + backward)" if training else ""
    big = cfg.B * cfg.N * cfg.H * cfg.D * cfg.elem_bytes
    names = "q, k, v, dO" if training else "q, k, v"
    return {"workload": f"{cfg.name}{variant}{what}: {cfg.describe()}", "seed": cfg.seed,
            "l2": (f"inputs larger than L2 ({names} {big / 1e6:.0f} MB each)" if big > 126e6 else
                   f"inputs smaller than L2 ({names} {big / 1e6:.1f} MB each), not flushed"),
            "parallelism": f"replica per GPU x{world}"}


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return
    q, k, v = W.make_inputs(cfg, device="cpu")
    heads = list(range(cfg.Hkv))
    causal = dict(causal=args.causal, force_diag=args.force_diag)
    for s in range(args.warmup):
        oracle_sample(q, k, v, cfg, [heads[s % cfg.Hkv]], 1, seed=100 + s, **causal)
    tok, sec, thr = 0, 0.0, 1
    for s in range(args.steps):
        t, dt, thr = oracle_sample(q, k, v, cfg, [heads[s % cfg.Hkv]], 1, seed=1000 + s, **causal)
        tok += t
        sec += dt
    value = tok / sec
    sample = (f"{args.steps} steps x 1 query block ({cfg.block_size * cfg.B * (cfg.H // cfg.Hkv)} tokens) "
              f"of one key/value head each, whole oracle path per step incl. pooling that head's k")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(cfg, args, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- training step

def run_backward(args, cfg, dev, rank, world, dist, bsa, flags, variant):
    """Times the training step: bsa_sparse_attn_fwd_train (the forward with
    lse) then bsa_sparse_attn_bwd, on the selection of the workload."""
    B, N, H, D, bs, ratio = cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size, cfg.topk_ratio
    kk = cfg.k
    q, k, v = W.make_inputs(cfg, device=dev)
    g = torch.Generator(device=dev).manual_seed(cfg.seed + 77)
    do = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(q.dtype)
    Hk = cfg.Hkv  # key/value heads (fewer than H with grouped queries)
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio, H_kv=Hk), device=dev, dtype=torch.uint8)
    bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws, flags=flags)  # the selection the step trains through
    idx = bsa.workspace_views(ws, B, N, H, D, bs, ratio, H_kv=Hk)[2].clone()
    bws = torch.empty(bsa.lib.bsa_sparse_attn_bwd_gqa_workspace_bytes(B, N, H, Hk, D, bs), device=dev,
                      dtype=torch.uint8)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        bsa.bsa_sparse_attn_fwd_train(q, k, v, idx, bs, flags=flags, out=o, lse=lse)
        if ev is not None:
            ev[1].record()
        grads = bsa.bsa_sparse_attn_bwd(q, k, v, o, do, idx, lse, bs, flags=flags, workspace=bws)
        if ev is not None:
            ev[2].record()
        return grads

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record()
    for s_ in range(args.steps):
        step(evs[s_])
    t1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t0.elapsed_time(t1)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    total_ms = max_over_ranks(total_ms, dist, dev)
    if bsa.bsa_device_error() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait")

    # end to end through the public API: host inputs in, gradients out
    hq, hk, hv, hdo = (x.cpu().pin_memory() for x in (q, k, v, do))
    hg = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (q, k, v)]  # dq, dk, dv
    dq_, dk_, dv_, ddo = (torch.empty_like(x) for x in (q, k, v, do))  # device copies of q, k, v, dO

    def e2e_step():
        for d_, h_ in ((dq_, hq), (dk_, hk), (dv_, hv), (ddo, hdo)):
            d_.copy_(h_, non_blocking=True)
        oo, ll = bsa.bsa_sparse_attn_fwd_train(dq_, dk_, dv_, idx, bs, flags=flags)
        grads = bsa.bsa_sparse_attn_bwd(dq_, dk_, dv_, oo, ddo, idx, ll, bs, flags=flags, workspace=bws)
        for h_, g_ in zip(hg, grads):
            h_.copy_(g_, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)

    flops_f = attn_flops(B, H, Hk, N, D, bs, kk, idx.cpu().numpy() if args.causal else None, args.causal)
    flops_b = 2.5 * flops_f  # five products of the forward's size (dS, dP recomputation not counted)
    peaks, peak_src = load_peaks()
    achieved = flops_b / (bwd_ms / 1e3) / 1e12
    nbytes = q.numel() * q.element_size()
    kvbytes = k.numel() * k.element_size()
    line = {
        "metric": METRIC, "value": job_tokens_per_s(B * N, world, args.steps, total_ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": workload_config(cfg, args, world, training=True),
        "gpu_launches": 5 * args.steps,
        "stages_ms": {"fwd_train": fwd_ms, "bwd": bwd_ms},
        "e2e": {"value": job_tokens_per_s(B * N, world, args.e2e_steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * nbytes + 2 * kvbytes, "d2h_bytes_per_step": nbytes + 2 * kvbytes,
                "steps": args.e2e_steps},
        "clocks": clk,
        "roofline": {"kernel": "bwd_dq_kernel + bwd_dkdv_kernel", "bound": "tensor", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} bf16 burst", "traffic": None,
                     "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                     "flops_per_launch": flops_b,
                     "forward_achieved": flops_f / (fwd_ms / 1e3) / 1e12},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        oracle.build()
        rng = np.random.default_rng(cfg.seed + 3000)
        il = idx.cpu().numpy()
        tok, sec = 0, 0.0
        for h in range(min(cfg.H, 2)):
            gk = h // (H // Hk)  # the query head's key/value head
            qa, da = (np.ascontiguousarray(W.to_oracle_array(x[:, :, h:h + 1])) for x in (q, do))
            ka, va = (np.ascontiguousarray(W.to_oracle_array(x[:, :, gk:gk + 1])) for x in (k, v))
            rows = np.sort(rng.choice(cfg.nb, size=(B, 1, 2), replace=False), axis=-1).astype(np.int32)
            t_ = time.perf_counter()
            oracle.sparse_attn_bwd(qa, ka, va, da, np.ascontiguousarray(il[:, gk:gk + 1]), bs, causal=args.causal,
                                   rows=rows)
            sec += time.perf_counter() - t_
            tok += 2 * bs * B
        line["cpu_baseline"] = {"value": tok / sec, "unit": "tokens/s", "cores": oracle.num_threads(),
                                "kind": "oracle",
                                "sample": f"backward of 2 random query blocks on each of {min(cfg.H, 2)} heads "
                                          f"({tok} query tokens, {sec:.1f} s)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our path

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c4", choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-blocks-per-head", type=int, default=8)
    ap.add_argument("--causal", action="store_true",
                    help="the causal variant (BSA_FLAG_CAUSAL): block-causal selection, token-causal attention")
    ap.add_argument("--force-diag", action="store_true",
                    help="with --causal: always keep the diagonal block (BSA_FLAG_FORCE_DIAG)")
    ap.add_argument("--dtype", choices=["bf16", "e4m3"], default=None,
                    help="override the config's input type (e4m3: FP8 inputs, bf16 output)")
    ap.add_argument("--kv-heads", type=int, default=None,
                    help="grouped queries: the config with this many key/value heads (H a multiple of it)")
    ap.add_argument("--backward", action="store_true",
                    help="time the training step (forward with lse + backward) instead of the forward")
    ap.add_argument("--stages-only", action="store_true",
                    help="time the stage-by-stage steps only (no fused, end-to-end or CPU legs); "
                         "for profiler runs")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.force_diag and not args.causal:
        ap.error("--force-diag needs --causal")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = W.CONFIGS[args.config]
    if args.dtype is not None:
        cfg = dataclasses.replace(cfg, dtype=args.dtype)
    if args.kv_heads is not None:
        if args.kv_heads < 1 or cfg.H % args.kv_heads:
            ap.error(f"--kv-heads must divide H={cfg.H}")
        cfg = dataclasses.replace(cfg, H_kv=args.kv_heads)

    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
        return

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    import block_sparse_attention_19_b200 as bsa

    flags = (bsa.BSA_FLAG_CAUSAL if args.causal else 0) | (bsa.BSA_FLAG_FORCE_DIAG if args.force_diag else 0)
    variant = (" causal" + (" force_diag" if args.force_diag else "")) if args.causal else ""
    if args.backward:
        run_backward(args, cfg, dev, rank, world, dist, bsa, flags, variant)
        if dist:
            dist.destroy_process_group()
        return

    B, N, H, D, bs, ratio = cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size, cfg.topk_ratio
    kk = bsa.bsa_topk_count(N // bs, ratio)
    q, k, v = W.make_inputs(cfg, device=dev)
    Hk = cfg.Hkv
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio, H_kv=Hk), device=dev,
                     dtype=torch.uint8)
    qp, kp, idx, S = bsa.workspace_views(ws, B, N, H, D, bs, ratio, with_scores=True, H_kv=Hk)
    o = torch.empty(q.shape, device=dev, dtype=torch.bfloat16 if cfg.dtype == "e4m3" else q.dtype)

    # one step: the selection stage (pooling of q and k in one launch, block
    # scores, top-k) then the attention, with an event around each stage; no
    # event between pooling and scoring, so that hand-off keeps the
    # programmatic-launch overlap bsa_forward has
    def step(ev=None):
        if ev is not None:
            ev[0].record()
        bsa.bsa_block_pool_qk(q, k, bs, q_out=qp, k_out=kp)
        bsa.bsa_block_scores_topk(qp, kp, kk, idx_out=idx, scores_out=S, flags=flags)
        if ev is not None:
            ev[1].record()
        bsa.bsa_sparse_attn_fwd(q, k, v, idx, bs, out=o, flags=flags)
        if ev is not None:
            ev[2].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if bsa.bsa_device_error() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start.record()
    for s in range(args.steps):
        step(evs[s])
    t_end.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    stage_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps  # selection stage
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    total_ms = max_over_ranks(total_ms, dist, dev)
    err = bsa.bsa_device_error()
    if err != 0:
        raise RuntimeError(f"a kernel gave up on a bounded wait (code {err})")
    # pooling alone (a diagnostic, after the timed steps): the same call K times
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record()
    for _ in range(args.steps):
        bsa.bsa_block_pool_qk(q, k, bs, q_out=qp, k_out=kp)
    p1.record()
    torch.cuda.synchronize()
    pool_ms = p0.elapsed_time(p1) / args.steps
    sel_ms = stage_ms - pool_ms  # scores and top-k, by difference

    if args.stages_only:
        if rank == 0:
            print(json.dumps({"stages_only": True, "config": cfg.name, "steps": args.steps,
                              "ms_per_step": total_ms / args.steps,
                              "stages_ms": {"selection": stage_ms, "pool_qk": pool_ms, "scores_topk": sel_ms,
                                            "sparse_attn": attn_ms}}),
                  flush=True)
        if dist:
            dist.destroy_process_group()
        return

    # ---- fused entry point, same inputs (reported beside the stage-by-stage step)
    fused_ms = None
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nf = max(3, args.steps // 4)
    f0.record()
    for _ in range(nf):
        bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws, out=o, flags=flags)
    f1.record()
    torch.cuda.synchronize()
    fused_ms = f0.elapsed_time(f1) / nf

    # ---- end to end through the host-buffer entry point: pinned host q, k, v
    # in, pinned host o out; the library copies head-group chunks in and out
    # on its own streams while earlier chunks compute
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hws = torch.empty(bsa.bsa_forward_host_workspace_bytes(B, N, H, D, bs, ratio, q.dtype, H_kv=Hk),
                      device=dev, dtype=torch.uint8)
    for _ in range(2):
        bsa.bsa_forward_host(hq, hk, hv, bs, ratio, out=ho, flags=flags, workspace=hws, synchronize=False)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.e2e_steps):
        bsa.bsa_forward_host(hq, hk, hv, bs, ratio, out=ho, flags=flags, workspace=hws, synchronize=False)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    if not torch.equal(ho, o.cpu()):
        raise RuntimeError("the host-buffer path disagrees with the device path")
    h2d = sum(x.numel() * x.element_size() for x in (q, k, v))
    d2h = o.numel() * o.element_size()
    del hq, hk, hv, ho, hws

    tokens_step = B * N
    value = job_tokens_per_s(tokens_step, world, args.steps, total_ms)
    e2e_value = job_tokens_per_s(tokens_step, world, args.e2e_steps, e2e_ms)
    flops = attn_flops(B, H, Hk, N, D, bs, kk, idx.cpu().numpy() if args.causal else None, args.causal)
    esz = cfg.elem_bytes
    tensor_bytes = B * N * H * D * esz  # q (and o)
    kv_bytes = B * N * Hk * D * esz     # k (and v): fewer heads with grouped queries
    idx_bytes = B * Hk * (N // bs) * kk * 4
    pooled_bytes = B * (H + Hk) * (N // bs) * D * 4
    o_bytes = B * N * H * D * (2 if cfg.dtype == "e4m3" else esz)  # e4m3 inputs give a bf16 output
    alg_bytes = tensor_bytes + o_bytes + 2 * kv_bytes + idx_bytes  # q, k, v read + o written, and the index list
    sel_bytes = tensor_bytes + kv_bytes + idx_bytes  # selection stage: q, k read + index list written
    peaks, peak_src = load_peaks()
    step_ms = total_ms / args.steps

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": workload_config(cfg, args, world),
        "tflops_effective": flops / (step_ms / 1e3) / 1e12,
        "gpu_launches": (4 if Hk == H else 5) * args.steps,
        "stages_ms": {"selection": stage_ms, "pool_qk": pool_ms, "scores_topk": sel_ms, "sparse_attn": attn_ms,
                      "fused_bsa_forward": fused_ms},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps},
        "clocks": clk,
    }
    if cfg.dtype in ("bf16", "e4m3"):
        # the tensor-core peak for the path's own type: FP8 takes the measured
        # bf16 peak times the nominal dense FP8 / bf16 ratio (4.5 / 2.25)
        mult = 2.0 if cfg.dtype == "e4m3" else 1.0
        peak, peak_sus = peaks["bf16_tflops"] * mult, peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * mult
        achieved = flops / (attn_ms / 1e3) / 1e12
        roof_t = max(flops / (peak * 1e12), alg_bytes / (peaks["hbm_gbs"] * 1e9))
        plain = not args.causal and Hk == H and cfg.dtype == "bf16"
        line["roofline"] = {
            "kernel": "sparse_attn_tc2_kernel",
            "bound": "tensor", "achieved": achieved,
            "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{peak_src} bf16 burst" + (" x 2 (nominal e4m3 / bf16 dense ratio)" if mult > 1 else ""),
            "traffic": NCU_TRAFFIC.get(cfg.name) if plain else None,
            "frac_of_sustained": achieved / peak_sus,
            "frac_of_roofline_time": roof_t / (attn_ms / 1e3),
            "flops_per_launch": flops, "algorithmic_bytes_per_launch": alg_bytes,
        }
        if bs == 64:
            # two query blocks share one 128 x 128 score tile, of which the
            # block-diagonal half is used: the score product runs twice its
            # algorithmic FLOPs. P.V does too with bf16 (one product over the
            # whole tile, the other block's half of P zero); with e4m3 it is
            # issued per block. So frac cannot exceed 0.5 (bf16) or 2/3 (e4m3).
            line["roofline"]["tensor_flops_per_launch"] = (1.5 if cfg.dtype == "e4m3" else 2.0) * flops
    line["selection_stage"] = {
        "bytes": sel_bytes, "ms": stage_ms,
        "GB/s": sel_bytes / (stage_ms / 1e3) / 1e9,
        "frac_of_hbm": sel_bytes / (stage_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "pool_GB/s": (tensor_bytes + kv_bytes + pooled_bytes) / (pool_ms / 1e3) / 1e9,
        "pool_frac_of_hbm": (tensor_bytes + kv_bytes + pooled_bytes) / (pool_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "peak": peaks["hbm_gbs"], "peak_source": f"{peak_src} HBM copy"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads = list(range(cfg.Hkv))
        qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
        bpe = min(args.cpu_blocks_per_head, cfg.nb)
        tok, sec, thr = oracle_sample(qc, kc, vc, cfg, heads, bpe, seed=cfg.seed + 2000,
                                      causal=args.causal, force_diag=args.force_diag)
        line["cpu_baseline"] = {"value": tok / sec, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                                "sample": f"{bpe} random query blocks on each of {len(heads)} key/value heads "
                                          f"({tok} query tokens, {sec:.1f} s), whole oracle path per head "
                                          f"incl. pooling all of that head's k"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
