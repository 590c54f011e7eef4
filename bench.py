#!/usr/bin/env python3
"""Benchmark of the fused, chunked distillation KL loss (forward + backward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kernels|reference]

One step = one kl_fwd_bwd call (top-K prep, logits + split-V statistics with the
fused cache gather, row merge, dS factors, dH and dW contractions that form dS
from the stored exponentials, loss mean) over one batch of the offline top-K
workload: N=4096 tokens, d=3072, V=128256, bf16, teacher cache K=64 (int32 ids +
fp32 logits + fp32 teacher log-sum-exp, partial mass kept), T=1.  Inputs are
synthetic and seeded; W (0.79 GB) and the logit chunk (1.05 GB) are larger than
the 126 MB L2, so no flush is needed between steps.  With --gpus N (under
torchrun) every rank runs its own N=4096-token shard, scaled by the global
count of valid tokens, and each step ends with the head gradient reduce-
scattered (or all-reduced, --dp-sync) and the loss all-reduced over NCCL (weak
scaling); the elapsed time is the max over ranks.

Prints ONE JSON line on rank 0.  `--impl reference` times the fp64 CPU oracle
instead, on the host cores, on a bounded row sample of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused KL fwd+bwd tokens/s at V=128256,d=3072; % bf16 TC peak; extra HBM GiB"
WORKLOAD = ("offline top-K KD: N=4096 tokens, d=3072, V=128256, bf16 H~N(0,1), "
            "W~N(0,0.02^2); cache K=64 int32 ids + fp32 logits + fp32 teacher lse "
            "(partial mass) from a bf16 teacher head d_t=4096; T=1")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kernels", choices=["kernels", "reference"])
    ap.add_argument("--workload", default="offline_topk",
                    choices=["offline_topk", "full_vocab", "packed_long", "scaling"])
    ap.add_argument("--N", type=int, default=0, help="tokens per GPU (0 = the workload's own)")
    ap.add_argument("--d", type=int, default=0,
                    help="offline top-K workload: student width (0 = the workload's 3072)")
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--reverse-weight", type=float, default=0.0,
                    help="teacher-hidden workload: weight of the reverse KL (0 = forward KL)")
    ap.add_argument("--entry", default="fused", choices=["fused", "split"],
                    help="fused: kl_fwd_bwd; split: kl_fwd then kl_bwd (the autograd path, "
                         "backward recomputes the logits)")
    ap.add_argument("--fuse-dlogits", action="store_true",
                    help="fused entry, bf16 top-K: form dS inside the dH contraction instead of "
                         "by a pass over the logit chunk (kl_problem.fuse_dlogits)")
    ap.add_argument("--recompute-all", action="store_true",
                    help="--entry split: the backward recomputes every chunk (by default, as "
                         "the autograd path, kl_fwd keeps the last chunk's logits for kl_bwd)")
    ap.add_argument("--parallel", default="tokens", choices=["tokens", "vocab"],
                    help="tokens: each rank its own token shard, no collective (weak scaling); "
                         "vocab: the head split by vocabulary rows over the ranks, the same "
                         "tokens on every rank, one statistics all-gather per chunk (two with "
                         "a reverse-KL weight) and an all-reduce of dH (strong scaling)")
    ap.add_argument("--dp-sync", default="reduce_scatter",
                    choices=["reduce_scatter", "all_reduce", "none"],
                    help="token shards on N>1 ranks: how each step combines the head gradient "
                         "(dW reduce-scattered into row blocks, as a sharded optimizer keeps it, "
                         "or all-reduced; the loss shares are all-reduced) -- 'none' times the "
                         "shards alone")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the short runs of the other benchmark configurations that the "
                         "default single-GPU line carries under 'secondary'")
    ap.add_argument("--cpu-sample", type=int, default=0,
                    help="tokens in the oracle sample (0 = sized to ~10 s)")
    return ap.parse_args()


WORKLOADS = {
    "offline_topk": WORKLOAD,
    "full_vocab": ("full-vocab recompute: N=8192, d=3072, teacher d_t=4096, V=128256, bf16 "
                   "hiddens N(0,1), heads N(0,0.02^2); teacher logits recomputed per chunk; T=2"),
    "packed_long": ("packed long context: N=32768 packed documents (lengths U[512,4096]), 5% of "
                    "positions masked; d=3072, V=128256, bf16, K=64 cache as offline top-K; T=1"),
    "scaling": ("output-head scaling sweep: offline top-K cache workload at the given N "
                "(4096/16384/65536/262144); d=3072, V=128256, bf16, K=64; T=1"),
}


def make_workload(wl, args, dev, rank):
    seed_shift = rank * 1000
    if args.workload == "offline_topk":
        return wl.offline_topk(device=dev, N=args.N or 4096, seed=1 + seed_shift, d=args.d or 3072)
    if args.workload == "full_vocab":
        return wl.full_vocab(device=dev, N=args.N or 8192, seed=2 + seed_shift)
    if args.workload == "packed_long":
        return wl.packed_long(device=dev, N=args.N or 32768, seed=3 + seed_shift)
    return wl.scaling(args.N or 262144, device=dev, seed=4 + seed_shift)


def problem_kwargs(w, chunk, override=None):
    o = override or {}
    kw = dict(T=w.T, mask=o.get("mask", w.mask), chunk_tokens=chunk)
    if w.mode == "topk":
        kw.update(topk_idx=o.get("topk_idx", w.topk_idx), topk_logit=o.get("topk_logit", w.topk_logit),
                  teacher_lse=o.get("teacher_lse", w.teacher_lse))
    else:
        kw.update(Ht=o.get("Ht", w.Ht), Wt=w.Wt)
    return kw


def _pg_timeout():
    import datetime

    return datetime.timedelta(seconds=int(os.environ.get("KL_BENCH_PG_TIMEOUT", "600")))


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def measured_peaks():
    """Roofline denominators: the measured peaks of this machine when
    MEASURED_PEAKS.json is present, else the pool's earlier measurement
    (copy 6.65 TB/s; cuBLAS bf16 1.59 PFLOP/s burst, about 1.4 sustained under
    the power cap)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        if all(isinstance(pk.get(k), (int, float)) for k in ("hbm_gbs", "bf16_tflops")):
            pk.setdefault("bf16_tflops_sustained", pk["bf16_tflops"])
            return pk, "measured"
    except Exception:
        pass
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
        "fallback"


# A timed region shorter than this runs on the burst clock: the kernels are
# compared with the burst GEMM figure; longer regions sit in the power cap and
# are compared with the sustained one.
BURST_REGION_S = 2.0


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        load = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def gpu_arm(args):
    import torch
    import torch.distributed as dist

    from chunked_kl_loss_tma_b200 import _lib, ops
    from chunked_kl_loss_tma_b200 import workloads as wl
    from chunked_kl_loss_tma_b200.dist import max_over_ranks

    ws, rank, local = dist_setup(args)
    local = local % max(torch.cuda.device_count(), 1)  # ranks beyond the devices share them
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        # KL_BENCH_BACKEND=gloo runs the same multi-rank path with host-side
        # collectives (e.g. several ranks sharing one GPU for a functional check)
        backend = os.environ.get("KL_BENCH_BACKEND", "nccl")
        if backend == "nccl":
            dist.init_process_group("nccl", device_id=dev, timeout=_pg_timeout())
        else:
            dist.init_process_group(backend, timeout=_pg_timeout())
    vocab = args.parallel == "vocab"
    if vocab and args.entry != "fused":
        raise SystemExit("--parallel vocab runs the fused pass (kl_vp_* calls)")
    # vocabulary-parallel ranks share the tokens: the same seed everywhere
    w = make_workload(wl, args, dev, 0 if vocab else rank)
    args.N = w.N
    torch.cuda.empty_cache()  # drop the teacher-cache generator's temporaries
    kw = problem_kwargs(w, args.chunk)
    if args.reverse_weight > 0:
        kw["reverse_weight"] = args.reverse_weight
    if args.fuse_dlogits:
        if args.entry != "fused":
            raise SystemExit("--fuse-dlogits applies to the fused entry (kl_fwd_bwd)")
        kw["fuse_dlogits"] = True
    shard = None
    dp_sync = args.dp_sync if (ws > 1 and not vocab) else "none"
    if vocab:
        from chunked_kl_loss_tma_b200 import vocab_parallel as vpm

        v0, v1 = vpm.vocab_shard(w.V, ws, rank)
        W_head = w.W[v0:v1]
        if w.mode == "hidden":
            kw["Wt"] = w.Wt[v0:v1]
        prob, keep = ops.make_problem(w.H, W_head, v_begin=v0, V_total=w.V, **kw)
    else:
        W_head = w.W
        if dp_sync != "none":
            # every rank scales by the batch's global count of valid tokens
            from chunked_kl_loss_tma_b200.dist import global_valid_count

            local = w.N if w.mask is None else int(w.mask.sum().item())
            kw["normalizer"] = float(global_valid_count(local))
        prob, keep = ops.make_problem(w.H, w.W, **kw)
    ws_bytes = ops.workspace_bytes(prob, _lib.KL_ENTRY_FWD_BWD)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    dH = torch.empty_like(w.H)
    dW = torch.empty(W_head.shape, dtype=torch.float32, device=dev)
    # extra HBM = everything allocated beyond inputs and gradients (the workspace)
    torch.cuda.synchronize()
    base_mem = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    if vocab:
        shard = vpm.ShardPass(w.H, W_head, v_begin=v0, V_total=w.V, dW=dW, workspace=workspace,
                              **kw)
        comm = vpm.TorchComm()

    if args.entry == "split":
        prob.keep_last_chunk = 0 if args.recompute_all else 1
        ws_split = max(ops.workspace_bytes(prob, _lib.KL_ENTRY_FWD),
                       ops.workspace_bytes(prob, _lib.KL_ENTRY_BWD))
        if ws_split > ws_bytes:
            workspace = torch.empty(ws_split, dtype=torch.uint8, device=dev)
            ws_bytes = ws_split
        lse_s = torch.empty(w.N, dtype=torch.float32, device=dev)
        lse_t = torch.empty(w.N, dtype=torch.float32, device=dev) if w.mode == "hidden" else None
        g_one = torch.ones((), dtype=torch.float32, device=dev)

    def dp_reduce():
        """Token shards: sum the head gradient over the ranks (reduce-scatter or
        all-reduce) and the loss shares."""
        from chunked_kl_loss_tma_b200.dist import reduce_scatter_rows, sum_over_ranks

        if dp_sync == "all_reduce":
            sum_over_ranks(dW)
        else:
            reduce_scatter_rows(dW)
        sum_over_ranks(loss.view(1))

    def step():
        if shard is not None:
            vpm.run_pass(shard, comm)
            return
        if args.entry == "split":
            _lib.check(_lib.kl_fwd(prob, workspace.data_ptr(), ws_bytes, loss.data_ptr(),
                                   lse_s.data_ptr(), None if lse_t is None else lse_t.data_ptr(),
                                   None, stream), "kl_fwd")
            _lib.check(_lib.kl_bwd(prob, workspace.data_ptr(), ws_bytes, lse_s.data_ptr(),
                                   None if lse_t is None else lse_t.data_ptr(), g_one.data_ptr(),
                                   dH.data_ptr(), dW.data_ptr(), 0, stream), "kl_bwd")
            return
        _lib.check(_lib.kl_fwd_bwd(prob, workspace.data_ptr(), ws_bytes, 1.0, loss.data_ptr(),
                                   None, dH.data_ptr(), dW.data_ptr(), 0, stream), "kl_fwd_bwd")
        if dp_sync != "none":
            dp_reduce()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    status = _lib.kl_status(workspace.data_ptr(), stream)
    if status != 0:
        raise RuntimeError(f"device status {_lib.STATUS.get(status)} after warm-up")

    def barrier():
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clocks.start()
    time.sleep(0.3)
    launches0 = _lib.kl_launch_count()
    _lib.kl_profile_begin()
    barrier()
    # one event after every step as well: the per-step distribution (median)
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e0.record()
    for i in range(args.steps):
        step()
        marks[i].record()
    e1.record()
    barrier()
    prof = _lib.kl_profile_end()
    launches = _lib.kl_launch_count() - launches0
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    per_step = sorted([e0.elapsed_time(marks[0])] +
                      [marks[i - 1].elapsed_time(marks[i]) for i in range(1, args.steps)])
    peak_extra = torch.cuda.max_memory_allocated(dev) - base_mem
    if ws > 1:
        ms = max_over_ranks(ms)

    # ---- end to end through the public API: pinned host inputs in, loss out.
    # Per-step inputs (hidden states, the teacher side, the mask) come from
    # pinned host memory every step; the heads stay resident (parameters).  A
    # double-buffered stager copies step i+1's inputs on its own stream while
    # step i's kernels run, and every step's loss is read back to pinned host
    # memory.  All copies of the K steps lie inside the timed region.
    e2e = None
    if not args.no_e2e and not vocab:
        from chunked_kl_loss_tma_b200.staging import HostStager

        names = ["H", "mask", "topk_idx", "topk_logit", "teacher_lse", "Ht"]
        host = {k: getattr(w, k).cpu().pin_memory() for k in names if getattr(w, k) is not None}
        stager = HostStager(host, dev, depth=2)
        probs = []
        for slot in range(stager.depth):
            kw2 = problem_kwargs(w, args.chunk, override=stager.bufs[slot])
            if args.reverse_weight > 0:
                kw2["reverse_weight"] = args.reverse_weight
            if args.fuse_dlogits:
                kw2["fuse_dlogits"] = True
            probs.append(ops.make_problem(stager.bufs[slot]["H"], w.W, **kw2))
        hloss = torch.empty(max(args.steps, 3), dtype=torch.float32).pin_memory()
        cstream = torch.cuda.current_stream(dev)

        def e2e_run(n):
            slot = stager.put(host)
            for i in range(n):
                stager.acquire(slot, cstream)
                nxt = stager.put(host) if i + 1 < n else None
                pr = probs[slot][0]
                if args.entry == "split":
                    pr.keep_last_chunk = prob.keep_last_chunk
                    _lib.check(_lib.kl_fwd(pr, workspace.data_ptr(), ws_bytes, loss.data_ptr(),
                                           lse_s.data_ptr(),
                                           None if lse_t is None else lse_t.data_ptr(), None,
                                           stream), "kl_fwd")
                    _lib.check(_lib.kl_bwd(pr, workspace.data_ptr(), ws_bytes, lse_s.data_ptr(),
                                           None if lse_t is None else lse_t.data_ptr(),
                                           g_one.data_ptr(), dH.data_ptr(), dW.data_ptr(), 0,
                                           stream), "kl_bwd")
                else:
                    _lib.check(_lib.kl_fwd_bwd(pr, workspace.data_ptr(), ws_bytes, 1.0,
                                               loss.data_ptr(), None, dH.data_ptr(),
                                               dW.data_ptr(), 0, stream), "kl_fwd_bwd")
                stager.release(slot, cstream)
                if dp_sync != "none":
                    dp_reduce()
                hloss[i].copy_(loss, non_blocking=True)
                slot = nxt

        e2e_run(3)
        barrier()
        e0.record()
        e2e_run(args.steps)
        e1.record()
        barrier()
        ems = e0.elapsed_time(e1)
        if ws > 1:
            ems = max_over_ranks(ems)
        e2e = {"value": ws * args.N * args.steps / (ems / 1e3),
               "unit": "tokens/s", "h2d_bytes_per_step": stager.bytes_per_step,
               "d2h_bytes_per_step": 4,
               "pipeline": "inputs double-buffered: step i+1's host-to-device copy overlaps "
                           "step i's kernels; loss read back every step"}

    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = measured_peaks()
    N, d, V = args.N, w.d, w.V
    tok_s = (1 if vocab else ws) * N * args.steps / (ms / 1e3)
    burst = ms / 1e3 < BURST_REGION_S
    peak_bf16 = peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]
    peak_desc = (f"{peak_src} {'burst' if burst else 'sustained'} bf16 GEMM "
                 f"(timed region {ms / 1e3:.2f} s {'<' if burst else '>='} {BURST_REGION_S} s)")
    dom = max(prof, key=lambda p: p["total_ms"]) if prof else None
    roof = None
    if dom is not None:
        per_launch_flops = dom["flops"] / max(dom["launches"], 1)
        avg_s = dom["total_ms"] / max(dom["launches"], 1) / 1e3
        if per_launch_flops > 0:
            achieved = per_launch_flops / avg_s / 1e12
            roof = {"kernel": dom["name"], "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": peak_bf16, "unit": "TFLOP/s", "frac": round(achieved / peak_bf16, 4),
                    "traffic": None, "peak_source": peak_desc,
                    "avg_launch_ms": round(avg_s * 1e3, 4),
                    "flops_per_launch": per_launch_flops}
        else:
            achieved = dom["bytes"] / max(dom["launches"], 1) / avg_s / 1e9
            roof = {"kernel": dom["name"], "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
                    "peak_source": f"{peak_src} copy bandwidth"}
        # DRAM counters need ncu, which never wraps a timed run: the per-launch
        # traffic of each kernel is in the committed ncu summaries instead.
        roof["traffic_note"] = "DRAM bytes per launch from ncu captures, not from this run"
        if roof["frac"] > 1.0:
            roof["frac_note"] = "above 1: the denominator does not match this run's clocks"
    # algorithmic tensor work per step: logits, dH and dW contractions (6 N d V),
    # plus the teacher logits (2 N d_t V) in the teacher-hidden mode
    step_flops = 6.0 * N * d * V + (2.0 * N * w.d_t * V if w.mode == "hidden" else 0.0)
    step_tflops = step_flops * args.steps / (ms / 1e3) / 1e12
    kernels = {p["name"]: {"launches": p["launches"], "ms": round(p["total_ms"], 3),
                           "share": round(p["total_ms"] / sum(q["total_ms"] for q in prof), 4)}
               for p in prof}
    line = {
        "metric": METRIC, "value": round(tok_s, 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "strong" if vocab else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init heads and teacher cache)",
        "config": {"workload": WORKLOADS[args.workload], "N_per_gpu": N, "d": d, "V": V,
                   "K": w.K or None, "d_t": w.d_t if w.mode == "hidden" else None, "T": w.T,
                   "masked_tokens": int((w.mask == 0).sum().item()) if w.mask is not None else 0,
                   "chunk_tokens": args.chunk or min(4096, N),
                   "l2": "inputs larger than L2 (W 0.79 GB, logit chunk 1.05 GB); no flush",
                   "parallelism": (f"vocabulary-parallel head shards x{ws}: all-gather of row "
                                   "statistics per chunk, all-reduce of fp32 dH"
                                   if vocab else
                                   f"weak-scaling token shards x{ws}, no data-path collective"
                                   if dp_sync == "none" else
                                   f"weak-scaling token shards x{ws}; per step the dW "
                                   f"{dp_sync.replace('_', '-')} and a loss all-reduce (NCCL)")},
        "entry": "kl_fwd_bwd" if args.entry == "fused" else "kl_fwd + kl_bwd (recompute)",
        "step_ms_median": round(per_step[len(per_step) // 2], 4),
        "step_ms_p10_p90": [round(per_step[len(per_step) // 10], 4),
                            round(per_step[(9 * len(per_step)) // 10], 4)],
        "tensor_tflops_step": round(step_tflops, 1),
        "tensor_frac_step": round(step_tflops / peak_bf16, 4),
        "tensor_frac_step_burst_peak": round(step_tflops / peaks["bf16_tflops"], 4),
        "tensor_frac_step_sustained_peak": round(step_tflops / peaks["bf16_tflops_sustained"], 4),
        "tensor_frac_step_spec_2250": round(step_tflops / 2250.0, 4),
        "extra_hbm_gib": round(ws_bytes / 2**30, 4),
        "extra_hbm_gib_measured_peak": round(peak_extra / 2**30, 4),
        "roofline": roof, "kernels": kernels, "gpu_launches": launches, "clocks": clk,
        "e2e": e2e,
    }
    if (ws == 1 and not args.no_secondary and args.workload == "offline_topk" and N == 4096
            and d == 3072 and args.entry == "fused" and not vocab and not args.fuse_dlogits):
        del workspace, dH, dW, keep, prob
        line["secondary"] = secondary_runs(dev, w)
    if not args.no_cpu_baseline and ws == 1:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_sample)
    if args.workload != "offline_topk":
        line["metric"] = METRIC + f" [{args.workload}]"
    elif args.d and args.d != 3072:
        line["metric"] = METRIC + f" [d={args.d}]"
    if args.fuse_dlogits:
        line["metric"] += " [dS formed in the dH contraction]"
        line["config"]["fuse_dlogits"] = True
    if args.reverse_weight > 0:
        line["metric"] += f" [reverse KL weight {args.reverse_weight}]"
        line["config"]["reverse_weight"] = args.reverse_weight
    if vocab:
        line["metric"] += " [vocabulary-parallel]"
        line["config"]["N_per_gpu"] = None
        line["config"]["N"] = N
    if args.entry == "split":
        line["metric"] += " [kl_fwd + kl_bwd]"
        line["config"]["keep_last_chunk"] = not args.recompute_all
        # backward recomputes the student (and teacher) logits of every chunk
        # (but the last one, when kept)
        C = args.chunk or 4096
        n_re = N if args.recompute_all else max(N - (N - 1) % C - 1, 0) if N > C else 0
        executed = step_flops + 2.0 * n_re * V * (d + (w.d_t if w.mode == "hidden" else 0))
        line["executed_tflops_step"] = round(executed * args.steps / (ms / 1e3) / 1e12, 1)
    print(json.dumps(line), flush=True)


SECONDARY = [
    # (name, workload kwargs, entry, timed steps)
    ("full_vocab_N8192", dict(kind="full_vocab"), "fused", 5),
    ("packed_long_N32768", dict(kind="packed_long"), "fused", 3),
    ("scaling_N16384", dict(kind="scaling", N=16384), "fused", 3),
    ("scaling_N65536", dict(kind="scaling", N=65536), "fused", 2),
    ("scaling_N262144", dict(kind="scaling", N=262144), "fused", 2),
    ("offline_topk_N4096_split", dict(kind="offline_topk"), "split", 10),
]


def secondary_runs(dev, main_w):
    """Short device-timed runs of the other benchmark configurations (the
    teacher-hidden, packed and scaling workloads, and the split kl_fwd + kl_bwd
    entry with the last chunk kept, as the autograd path runs it), so that one
    default run records every configuration.  Each: 2 warm-up steps, then a few
    steps timed with CUDA events on the launch stream; inputs resident in HBM
    and larger than L2."""
    import torch

    from chunked_kl_loss_tma_b200 import _lib, ops
    from chunked_kl_loss_tma_b200 import workloads as wl

    out = {}
    stream = torch.cuda.current_stream(dev).cuda_stream
    for name, spec, entry, steps in SECONDARY:
        kind = spec["kind"]
        if kind == "offline_topk":
            w = main_w
        elif kind == "full_vocab":
            w = wl.full_vocab(device=dev)
        elif kind == "packed_long":
            w = wl.packed_long(device=dev)
        else:
            w = wl.scaling(spec["N"], device=dev)
        torch.cuda.empty_cache()
        kw = problem_kwargs(w, 0)
        prob, keep = ops.make_problem(w.H, w.W, **kw)
        if entry == "split":
            prob.keep_last_chunk = 1
        wsb = ops.workspace_bytes(prob, _lib.KL_ENTRY_FWD_BWD)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        loss = torch.empty((), dtype=torch.float32, device=dev)
        dH = torch.empty_like(w.H)
        dW = torch.empty(w.W.shape, dtype=torch.float32, device=dev)
        lse_s = torch.empty(w.N, dtype=torch.float32, device=dev)
        g_one = torch.ones((), dtype=torch.float32, device=dev)

        def step():
            if entry == "split":
                _lib.check(_lib.kl_fwd(prob, ws.data_ptr(), wsb, loss.data_ptr(), lse_s.data_ptr(),
                                       None, None, stream), "kl_fwd")
                _lib.check(_lib.kl_bwd(prob, ws.data_ptr(), wsb, lse_s.data_ptr(), None,
                                       g_one.data_ptr(), dH.data_ptr(), dW.data_ptr(), 0, stream),
                           "kl_bwd")
            else:
                _lib.check(_lib.kl_fwd_bwd(prob, ws.data_ptr(), wsb, 1.0, loss.data_ptr(), None,
                                           dH.data_ptr(), dW.data_ptr(), 0, stream), "kl_fwd_bwd")

        for _ in range(2):
            step()
        torch.cuda.synchronize()
        status = _lib.kl_status(ws.data_ptr(), stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            step()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        flops = 6.0 * w.N * w.d * w.V + (2.0 * w.N * w.d_t * w.V if w.mode == "hidden" else 0.0)
        out[name] = {"tokens_per_s": round(w.N / (ms / 1e3), 1), "ms_per_step": round(ms, 3),
                     "steps": steps, "entry": "kl_fwd + kl_bwd (last chunk kept)"
                     if entry == "split" else "kl_fwd_bwd",
                     "useful_tflops": round(flops / (ms / 1e3) / 1e12, 1),
                     "frac_of_spec_2250": round(flops / (ms / 1e3) / 1e12 / 2250.0, 4),
                     "extra_hbm_gib": round(wsb / 2**30, 4), "status": status,
                     "loss": round(float(loss.item()), 6)}
        del prob, keep, ws, dH, dW, lse_s
        if w is not main_w:
            del w
        torch.cuda.empty_cache()
    return out


def _oracle_sample(w, n_tokens):
    """The oracle on the first n_tokens rows of the workload as a problem of its
    own (loss, dH and dW over those rows)."""
    import oracle

    sl = slice(0, n_tokens)
    kw = dict(T=w.T, mode=w.mode, mask=None if w.mask is None else w.mask[sl])
    if w.mode == "topk":
        kw.update(topk_idx=w.topk_idx[sl], topk_logit=w.topk_logit[sl],
                  teacher_lse=None if w.teacher_lse is None else w.teacher_lse[sl])
    else:
        kw.update(Ht=w.Ht[sl], Wt=w.Wt)
    return oracle.kl_loss(w.H[sl], w.W, **kw)


def _cores():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline(w, n_tokens=0, target_s=10.0):
    """fp64 oracle throughput on the host cores over a bounded token sample,
    sized from two short probes to about target_s seconds of CPU work."""
    sample = w.to("cpu")
    if n_tokens <= 0:
        t0 = time.time()
        _oracle_sample(sample, 8)
        t8 = time.time() - t0
        t0 = time.time()
        _oracle_sample(sample, 40)
        t40 = time.time() - t0
        per_token = max((t40 - t8) / 32, 1e-6)
        fixed = max(t8 - 8 * per_token, 0.0)
        n_tokens = int(min(max((target_s - fixed) / per_token, 16), 4096, w.N))
    t0 = time.time()
    _oracle_sample(sample, n_tokens)
    dt = time.time() - t0
    return {"value": round(n_tokens / dt, 3), "unit": "tokens/s", "cores": _cores(),
            "kind": "oracle",
            "sample": f"first {n_tokens} tokens of the workload as a problem of their own "
                      f"(fp64 loss, dH and dW; {dt:.1f} s)"}


def reference_arm(args):
    ws, rank, local = dist_setup(args)
    if rank != 0:
        return
    import torch

    from chunked_kl_loss_tma_b200 import workloads as wl

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = make_workload(wl, args, dev, 0).to("cpu")
    args.N = w.N
    # Each oracle call pays a fixed cost (the fp64 [V, d] dW it returns is
    # zeroed and written once), so a step of a few rows measures that cost, not
    # per-token work: 256 rows keep it a minor part while a 20-step run stays
    # within a couple of minutes.
    per_step = args.cpu_sample or 256
    for _ in range(max(args.warmup, 3)):
        _oracle_sample(w, 2)
    t0 = time.time()
    for _ in range(args.steps):
        _oracle_sample(w, per_step)
    dt = time.time() - t0
    v = per_step * args.steps / dt
    metric = METRIC + ("" if args.workload == "offline_topk" else f" [{args.workload}]")
    line = {
        "impl": "reference", "metric": metric, "value": round(v, 3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOADS[args.workload], "N_per_gpu": w.N,
                   "sample_per_step": f"{per_step} tokens (fp64 oracle on host cores)"},
        "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": _cores(),
                         "kind": "oracle",
                         "sample": f"{per_step} tokens per step of the same workload"},
        "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
