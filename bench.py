"""Benchmark of the MoE routing hot path on B200: routed tokens/s.

One step = the whole path over one batch of T tokens, every stage a libmr.so
kernel launched through the C ABI on one stream:
    router (3xTF32 tcgen05 GEMM + fused routing)  -> idx, w
    dispatch (counts, offsets, stable perm, inv)   -> perm, inv
    gather (token rows -> expert-sorted rows)      -> xs [T*k, d]
    [expert FFNs are not part of the path: synthetic expert outputs E]
    combine (weighted sum + shared add)            -> y [T, d]
Default workload: the full DeepSeek-V3 routing + dispatch + combine batch
(T=16384, d=7168, 256 experts in 8 groups keep 4, top-8, bf16 rows).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (one rank per GPU, under torchrun, or started by this script when
--gpus N > 1 is given without a launcher): every rank runs its own batch
(replicas, weak scaling, no collective in the data path); value = all ranks'
tokens / max-over-ranks device time.  --impl reference times the CPU oracle
(rank 0 only) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "routed tokens/sec (router+dispatch+combine) at 1 B200; % of roofline"
UNIT = "tokens/s"

# B200 peer-to-peer copy bandwidth per direction over NVLink 5 / NVSwitch
# (measured copy; 900 GB/s nominal): the bound of rows crossing to other GPUs.
NVLINK_PEER_GBS = 770.0

# DRAM traffic per launch measured with ncu (dram__bytes_read.sum +
# dram__bytes_write.sum) for the dominant kernel, keyed by the SHA-256 of the
# source file it was built from; reported only while the source is unchanged.
NCU_TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum of the current
    # source on the full DeepSeek-V3 batch (T=16384; one pass per launch; the
    # mean of four launches at 16 CTAs per SM): 2115.01 MB read + 226.01 MB
    # written per launch.
    "combine": {"src": "f0e65656306c92ab", "bytes": 2115013312 + 226008384},
}


def _src_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons (read-only)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

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
                if len(parts) < 9:
                    continue
                try:
                    rows.append({"sm": float(parts[2]), "max": float(parts[3]),
                                 "hw": parts[5], "hwt": parts[6], "swt": parts[7],
                                 "pcap": parts[8]})
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r["sm"] for r in rows])),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the reference arm)

def _oracle_sample(w: wl.Workload, n_tok: int, inputs, threads=0):
    """One pass of the oracle over n_tok tokens of the workload: router on
    their rows, dispatch of their k*n_tok assignments, gather and combine of
    their rows (threads = 0: every host thread).  Returns the seconds it
    took."""
    import oracle
    x, W, b = inputs["x_f32"][:n_tok], inputs["W"], inputs["b"]
    rows = inputs["x_rows"][:n_tok]
    E, sh = inputs["E"][: n_tok * w.k], inputs["shared"][:n_tok]
    t0 = time.perf_counter()
    r = oracle.router(x, W, b, w.n_group, w.topk_group, w.k, w.route_scale, w.mask_mode,
                      threads=threads)
    _, _, perm, inv = oracle.dispatch(r["idx"], w.N_r)
    oracle.gather(rows, w.k, perm)
    oracle.combine(E, r["w"].astype(np.float32), inv, sh, w.k, threads=threads)
    return time.perf_counter() - t0


def _oracle_inputs(w: wl.Workload, n_tok: int):
    sub = w.replace(T=n_tok)
    d = wl.gen_router_inputs(w.replace(T=n_tok))
    return {"x_f32": d["x_f32"], "W": d["W"], "b": d["b"],
            "x_rows": d["x_bf16"] if w.io_dtype == "bf16" else d["x_f32"],
            "E": wl.gen_E(sub), "shared": wl.gen_shared(sub)}


def _router_check(w: wl.Workload, gpu_router):
    """The oracle's router over every token of the workload (rank 0's batch),
    timed, with its near-tie count and the GPU's selection compared outside
    the near-ties (gpu_router = (idx, w) of the timed step)."""
    import oracle
    d = wl.gen_router_inputs(w)
    t0 = time.perf_counter()
    r = oracle.router(d["x_f32"], d["W"], d["b"], w.n_group, w.topk_group, w.k, w.route_scale,
                      w.mask_mode)
    secs = time.perf_counter() - t0
    m = r["margins"]
    msel = np.minimum(m[:, 0], m[:, 1])
    tie = (msel <= oracle.NEAR_TIE_EPS) & (msel > 0)
    otie = tie | ((m[:, 2] <= oracle.NEAR_TIE_EPS) & (m[:, 2] > 0))
    gidx, gw = gpu_router
    ok = ~tie
    bad = int((np.sort(gidx, 1) != np.sort(r["idx"], 1)).any(1)[ok].sum())
    og, orr = np.argsort(gidx, 1, kind="stable"), np.argsort(r["idx"], 1, kind="stable")
    wg = np.take_along_axis(gw.astype(np.float64), og, 1)[ok]
    wr = np.take_along_axis(r["w"], orr, 1)[ok]
    return {"tokens": int(w.T), "near_ties": int(tie.sum()), "order_ties": int(otie.sum()),
            "selection_mismatches_outside_near_ties": bad,
            "w_max_rel_outside_near_ties": float((np.abs(wg - wr) / np.abs(wr)).max()),
            "eps": oracle.NEAR_TIE_EPS,
            "source": "fp64 oracle router over every token of the benchmark batch, against "
                      "the GPU's idx/w of the timed step"}, secs


def cpu_baseline(w: wl.Workload, target_s=15.0, gpu_router=None):
    """The oracle on a bounded sample of the workload: passes over the same
    `cap` tokens until about target_s seconds of CPU work have run.  With
    gpu_router, also the oracle's router over the whole batch (timed, with
    the near-tie count and a check of the GPU's selection: "router_check")."""
    import oracle
    check = None
    if gpu_router is not None:
        check, secs = _router_check(w, gpu_router)
        check["oracle_router_s"] = secs
        check["oracle_router_tokens_per_s"] = w.T / secs
    cap = 2048
    inp = _oracle_inputs(w, cap)
    t = _oracle_sample(w, 64, inp)
    n = int(min(cap, max(64, 64 * target_s / max(t, 1e-3))))
    passes = max(1, int(round(target_s / max(t * n / 64, 1e-3))))
    total = sum(_oracle_sample(w, n, inp) for _ in range(passes))
    # the same oracle on one host thread, over a quarter of the sample
    n1 = max(16, n // 4)
    t1 = _oracle_sample(w, n1, inp, threads=1)
    out = {"value": n * passes / total, "unit": UNIT, "cores": oracle.num_threads(),
           "kind": "oracle",
           "value_single_thread": n1 / t1,
            "sample": f"{passes} pass(es) over {n} tokens of {w.name} through the fp64 oracle "
                      f"(router, dispatch, gather, combine), {total:.1f} s; single thread: "
                      f"{n1} tokens, {t1:.1f} s"}
    if check is not None:
        out["router_check"] = check
    return out


def run_reference(args, w: wl.Workload, rank: int):
    if rank != 0:
        return
    import oracle
    probe = _oracle_sample(w, 16, _oracle_inputs(w, 16))
    per_step_s = 150.0 / max(1, args.steps + args.warmup)  # whole run within minutes
    n = int(min(512, max(8, 16 * min(per_step_s, 6.0) / max(probe, 1e-3))))
    inp = _oracle_inputs(w, n)
    for _ in range(args.warmup):
        _oracle_sample(w, n, inp)
    times = [_oracle_sample(w, n, inp) for _ in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, extra={"sample_tokens_per_step": n,
                                    "router_precision": "fp64 oracle (CPU)"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{n} tokens of {w.name} per step (fp64 oracle: router, "
                                   f"dispatch, gather, combine)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(w: wl.Workload, extra=None):
    c = {"workload": w.name, "T": w.T, "d": w.d, "N_r": w.N_r, "n_group": w.n_group,
         "topk_group": w.topk_group, "k": w.k, "route_scale": w.route_scale,
         "mask": "-inf" if w.mask_mode == wl.MASK_NEG_INF else "zero",
         "rows_dtype": w.io_dtype,
         "router_precision": ("bf16x3: bf16 rows x three bf16 planes of W, exact products, "
                              "fp32 accumulation (tcgen05 kind::f16)")
         if w.io_dtype == wl.BF16 else "3xTF32 (tcgen05 kind::tf32)",
         "l2": "inputs larger than L2 (x 235 MB + E 1.88 GB + shared 235 MB per step)",
         "parallelism": "replicas (token batches per GPU, no collective)"}
    if extra:
        c.update(extra)
    return c


# ---------------------------------------------------------------------------
# Multi-rank host logic (replicas): each rank routes its own seeded batch; the
# step time is the max over ranks; the value counts every rank's tokens.

def rank_workload(w: wl.Workload, rank: int) -> wl.Workload:
    """The batch rank `rank` routes: the same shapes, its own seed."""
    return w.replace(seed=w.seed + 1000 * rank)


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Max of a per-rank time over all ranks (all_reduce MAX when world > 1)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(world: int, T: int, ms_max: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return world * T / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# GPU arm

def run_router_only(args, w: wl.Workload):
    """The router stage alone on the workload (a profiling aid: ncu captures
    of the router run this), in the benchmark's launch configuration: bf16
    rows above 256 tokens through mr_router_forward_ex (bf16x3, workspace);
    otherwise the plain entry point on fp32 rows.  --router-weights bf16
    times mr_router_forward_bf16w instead.  Prints one JSON line."""
    import torch

    import token_dispatch_fp32_b200 as mr
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    d = wl.gen_router_inputs(w)
    bf16_rows = w.io_dtype == wl.BF16
    x32 = torch.from_numpy(d["x_f32"]).to(dev)
    xb = torch.from_numpy(d["x_bf16"]).view(torch.bfloat16).to(dev) if bf16_rows else None
    Wd = torch.from_numpy(d["W"]).to(dev)
    Wb = torch.from_numpy(wl.gen_W_bf16(w)["W_bf16"]).view(torch.bfloat16).to(dev)
    bd = torch.from_numpy(d["b"]).to(dev)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    wt = torch.empty((w.T, w.k), dtype=torch.float32, device=dev)
    ws = torch.empty(max(4, mr.mr_router_workspace_size(w.T, w.d, w.N_r)), dtype=torch.uint8,
                     device=dev)
    if args.router_weights == "bf16":
        how = "mr_router_forward_bf16w (bf16 rows, bf16 W)"

        def call():
            mr.mr_router_forward_bf16w(xb if bf16_rows else x32, Wb, bd, w.n_group, w.topk_group,
                                       w.k, w.route_scale, w.mask_mode, idx_out=idx, w_out=wt,
                                       workspace=ws, stream=stream)
    elif bf16_rows and w.T > 256:
        how = "mr_router_forward_ex (bf16 rows, bf16x3)"

        def call():
            mr.mr_router_forward_ex(xb, Wd, bd, w.n_group, w.topk_group, w.k, w.route_scale,
                                    w.mask_mode, precision=mr.MR_PREC_BF16X3, idx_out=idx,
                                    w_out=wt, workspace=ws, stream=stream)
    else:
        how = "mr_router_forward (fp32 rows)"

        def call():
            mr.mr_router_forward(x32, Wd, bd, w.n_group, w.topk_group, w.k, w.route_scale,
                                 w.mask_mode, idx_out=idx, w_out=wt, stream=stream)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0 = mr.mr_launch_count()
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    assert mr.mr_get_error(stream) == mr.MR_OK
    ms = e0.elapsed_time(e1) / args.steps
    fl = 2.0 * w.T * w.d * w.N_r
    print(json.dumps({"only": "router", "workload": w.name, "entry_point": how,
                      "ms": ms, "steps": args.steps, "warmup": args.warmup,
                      "launches_per_call": (mr.mr_launch_count() - l0) / args.steps,
                      "tflops_algorithmic": fl / (ms / 1e3) / 1e12,
                      "tc_cluster_pin": os.environ.get("MR_TC_CLUSTER"),
                      "l2": "back-to-back calls (inputs of the full workloads exceed L2)"}),
          flush=True)


def run_expert_only(args, w: wl.Workload):
    """The gather-fused expert layer alone (a profiling aid): route and
    dispatch the workload, then time mr_expert_gemm_gather with --n-out
    output columns per expert.  Prints one JSON line."""
    import torch

    import token_dispatch_fp32_b200 as mr
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    d = wl.gen_router_inputs(w)
    xb = torch.from_numpy(d["x_bf16"]).view(torch.bfloat16).to(dev)
    ws = torch.empty(max(4, mr.mr_router_workspace_size(w.T, w.d, w.N_r)), dtype=torch.uint8,
                     device=dev)
    idx, wt = mr.mr_router_forward_ex(xb, torch.from_numpy(d["W"]).to(dev),
                                      torch.from_numpy(d["b"]).to(dev), w.n_group,
                                      w.topk_group, w.k, w.route_scale, w.mask_mode,
                                      precision=mr.MR_PREC_BF16X3, workspace=ws, stream=stream)
    _, offsets, perm, _ = mr.mr_dispatch(idx, w.N_r, stream=stream)
    eW = torch.from_numpy(wl.gen_expert_W(w, args.n_out)).view(torch.bfloat16).to(dev)
    out = torch.empty((w.T * w.k, args.n_out), dtype=torch.bfloat16, device=dev)
    eWp = mr.mr_expert_pack_weights(eW, stream=stream) if args.expert_weights == "packed" \
        else None
    rows, rperm = xb, perm
    if args.expert_rows == "sorted":  # the rows materialised first; the GEMM alone is timed
        rows = mr.mr_gather_rows(xb, w.k, perm=perm, stream=stream)
        rperm = None

    if args.expert_epilogue == "combine":
        if rperm is None:
            raise SystemExit("--expert-epilogue combine needs --expert-rows gather")
        gen = torch.Generator(device=dev)
        gen.manual_seed(w.seed + 1)
        csh = torch.randn((w.T, args.n_out), generator=gen, device=dev).to(torch.bfloat16)
        cacc = torch.empty((w.T, args.n_out), dtype=torch.float32, device=dev)
        cy = torch.empty((w.T, args.n_out), dtype=torch.bfloat16, device=dev)

    def call():
        if args.expert_epilogue == "combine":
            mr.mr_expert_gemm_gather_combine(
                rows, w.k, rperm, offsets, eWp if eWp is not None else eW, wt, csh, N_r=w.N_r,
                n_out=args.n_out, packed=eWp is not None, acc=cacc, y=cy, stream=stream)
        elif eWp is not None:
            mr.mr_expert_gemm_gather_packed(rows, w.k, rperm, offsets, eWp, w.N_r, args.n_out,
                                            out=out, stream=stream)
        else:
            mr.mr_expert_gemm_gather(rows, w.k, rperm, offsets, eW, out=out, stream=stream)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    assert mr.mr_get_error(stream) == mr.MR_OK
    ms = e0.elapsed_time(e1) / args.steps
    fl = 2.0 * w.T * w.k * w.d * args.n_out
    print(json.dumps({"only": "expert", "workload": w.name, "n_out": args.n_out, "ms": ms,
                      "weights": args.expert_weights, "rows": args.expert_rows,
                      "epilogue": args.expert_epilogue,
                      "tflops": fl / (ms / 1e3) / 1e12, "steps": args.steps}), flush=True)


def run_ours(args, w: wl.Workload, rank: int, world: int):
    import torch
    import torch.distributed as dist

    import token_dispatch_fp32_b200 as mr

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(dev)

    # inputs (seeded per rank; every rank routes its own batch)
    wr = rank_workload(w, rank)
    d = wl.gen_router_inputs(wr)
    bf16_rows = w.io_dtype == wl.BF16
    x32 = torch.from_numpy(d["x_f32"]).to(dev)
    xb = torch.from_numpy(d["x_bf16"]).view(torch.bfloat16).to(dev) if bf16_rows else x32
    row_t = torch.bfloat16 if bf16_rows else torch.float32
    Wd = torch.from_numpy(d["W"]).to(dev)
    bd = torch.from_numpy(d["b"]).to(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wr.seed)
    E = torch.randn((w.T * w.k, w.d), generator=gen, device=dev, dtype=torch.float32).to(row_t)
    shared = torch.randn((w.T, w.d), generator=gen, device=dev, dtype=torch.float32).to(row_t)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    wt = torch.empty((w.T, w.k), dtype=torch.float32, device=dev)
    counts = torch.empty(w.N_r, dtype=torch.int32, device=dev)
    offsets = torch.empty(w.N_r + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(w.T * w.k, dtype=torch.int32, device=dev)
    inv = torch.empty(w.T * w.k, dtype=torch.int32, device=dev)
    xs = torch.empty((w.T * w.k, w.d), dtype=row_t, device=dev)
    y = torch.empty((w.T, w.d), dtype=row_t, device=dev)
    ws_r = torch.empty(max(4, mr.mr_router_workspace_size(w.T, w.d, w.N_r)), dtype=torch.uint8,
                       device=dev)
    ws_d = torch.empty(max(4, mr.mr_dispatch_workspace_size(w.T, w.k, w.N_r)),
                       dtype=torch.uint8, device=dev)

    names = ("router", "dispatch", "gather", "combine")
    # The router reads the hidden states as stored (bf16 rows: the bf16x3
    # tensor-core decomposition, exact products); fp32 rows take 3xTF32.
    router_prec = mr.MR_PREC_BF16X3 if bf16_rows else mr.MR_PREC_3XTF32

    def router(xin, prec, idx_out=idx, w_out=wt):
        mr.mr_router_forward_ex(xin, Wd, bd, w.n_group, w.topk_group, w.k, w.route_scale,
                                w.mask_mode, precision=prec, idx_out=idx_out, w_out=w_out,
                                workspace=ws_r, stream=stream)

    # one step's inputs (token rows, expert outputs, shared-expert output) and
    # results (idx, w, y); the end-to-end leg below alternates two such sets
    main_set = {"x": xb, "E": E, "shared": shared, "idx": idx, "wt": wt, "y": y}

    def step(ev=None, bufs=main_set):
        if ev is not None:
            ev[0].record(stream)
        router(bufs["x"], router_prec, bufs["idx"], bufs["wt"])
        if ev is not None:
            ev[1].record(stream)
        mr.mr_dispatch(bufs["idx"], w.N_r, counts=counts, offsets=offsets, perm=perm,
                       inv_perm=inv, workspace=ws_d, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        mr.mr_gather_rows(bufs["x"], w.k, perm=perm, inv_perm=inv, xs=xs, stream=stream)
        if ev is not None:
            ev[3].record(stream)
        mr.mr_combine(bufs["E"], bufs["wt"], inv, bufs["shared"], y=bufs["y"], stream=stream)
        if ev is not None:
            ev[4].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert mr.mr_get_error(stream) == mr.MR_OK

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = Clocks(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize(dev)
    l0 = mr.mr_launch_count()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    launches = mr.mr_launch_count() - l0
    barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end) / args.steps
    stage_ms = {n: float(np.mean([e[j].elapsed_time(e[j + 1]) for e in evs]))
                for j, n in enumerate(names)}
    assert mr.mr_get_error(stream) == mr.MR_OK
    step_router_out = (idx.cpu().numpy(), wt.cpu().numpy())  # checked by the oracle leg

    ms_max = max_over_ranks(ms, world, dev)

    # ---- router variants and other router shapes, each timed alone ----------
    # Between timed calls a read pass over a buffer of 4x the L2 leaves the L2
    # holding clean lines of that buffer, so every call reads its inputs from
    # HBM without paying for dirty-line write-backs.
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush.fill_(1)
    flush_i32 = flush.view(torch.int32)

    def read_flush():
        with torch.cuda.stream(stream):
            flush_i32.sum(dtype=torch.int64)

    def write_flush():
        with torch.cuda.stream(stream):
            flush.fill_(1)

    alone_means = {}

    def time_alone(fn, n, flush_fn=read_flush):
        """Median device time (ms) of fn() on the stream over n calls, each
        after flush_fn (events bracket fn alone); the mean is kept in
        alone_means[fn]."""
        for _ in range(3):
            fn()
        ts = []
        for _ in range(n):
            if flush_fn is not None:
                flush_fn()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        alone_means[fn] = float(np.mean(ts))
        return float(np.median(ts))

    n_alone = max(10, min(50, args.steps))
    # The router on the fp32 cast of the same rows: 3xTF32 (three tf32
    # products) and plain TF32 (one product, reported separately).
    alt_ms = tf32_ms = None
    if bf16_rows:
        alt_ms = time_alone(lambda: router(x32, mr.MR_PREC_3XTF32), n_alone, None)
        tf32_ms = time_alone(lambda: router(x32, mr.MR_PREC_TF32), n_alone, None)

    # The DeepSeek-V3 and Kimi K2 prefill routers (4096 and 8192 tokens), in
    # the benchmark's arithmetic (bf16 rows, bf16x3), timed alone.
    other_routers = {}
    if args.workload == wl.V3_FULL.name and not args.no_extra_stages:
        for key, wo in (("router_deepseek_v3_prefill_T4096", wl.V3_PREFILL),
                        ("router_kimi_k2_prefill_T8192", wl.K2_PREFILL)):
            oin = wl.gen_router_inputs(wo)
            ox = torch.from_numpy(oin["x_bf16"]).view(torch.bfloat16).to(dev)
            oW = torch.from_numpy(oin["W"]).to(dev)
            ob = torch.from_numpy(oin["b"]).to(dev)
            oidx = torch.empty((wo.T, wo.k), dtype=torch.int32, device=dev)
            owt = torch.empty((wo.T, wo.k), dtype=torch.float32, device=dev)
            ows = torch.empty(max(4, mr.mr_router_workspace_size(wo.T, wo.d, wo.N_r)),
                              dtype=torch.uint8, device=dev)

            def orouter(wo=wo, ox=ox, oW=oW, ob=ob, oidx=oidx, owt=owt, ows=ows):
                mr.mr_router_forward_ex(ox, oW, ob, wo.n_group, wo.topk_group, wo.k,
                                        wo.route_scale, wo.mask_mode,
                                        precision=mr.MR_PREC_BF16X3, idx_out=oidx, w_out=owt,
                                        workspace=ows, stream=stream)

            oms = time_alone(orouter, n_alone)
            of = 2.0 * wo.T * wo.d * wo.N_r
            other_routers[key] = {"workload": wo.name, "ms": oms,
                                  "tflops_algorithmic": of / (oms / 1e3) / 1e12,
                                  "tflops_issued": 3 * of / (oms / 1e3) / 1e12,
                                  "l2": "read pass over 512 MB before each call"}
            del ox, oW, ob, oidx, owt, ows
        assert mr.mr_get_error(stream) == mr.MR_OK

    # One synthetic expert layer (d -> 2048, the DeepSeek-V3 expert width) over
    # the expert-sorted rows of the DeepSeek-V3 prefill batch, with the row
    # gather fused into the grouped GEMM; beside it the unfused pair (the
    # sorted rows written by mr_gather_rows, then the same GEMM reading them
    # through an identity permutation).
    expert = None
    if args.workload == wl.V3_FULL.name and not args.no_extra_stages:
        we, n_out = wl.V3_PREFILL, 2048
        ein = wl.gen_router_inputs(we)
        ex = torch.from_numpy(ein["x_bf16"]).view(torch.bfloat16).to(dev)
        ews = torch.empty(max(4, mr.mr_router_workspace_size(we.T, we.d, we.N_r)),
                          dtype=torch.uint8, device=dev)
        eidx, ewt = mr.mr_router_forward_ex(ex, torch.from_numpy(ein["W"]).to(dev),
                                            torch.from_numpy(ein["b"]).to(dev), we.n_group,
                                            we.topk_group, we.k, we.route_scale, we.mask_mode,
                                            precision=mr.MR_PREC_BF16X3, workspace=ews,
                                            stream=stream)
        ecounts, eoff, eperm, einv = mr.mr_dispatch(eidx, we.N_r, stream=stream)
        eW = torch.from_numpy(wl.gen_expert_W(we, n_out)).view(torch.bfloat16).to(dev)
        eout = torch.empty((we.T * we.k, n_out), dtype=torch.bfloat16, device=dev)
        exs = torch.empty((we.T * we.k, we.d), dtype=torch.bfloat16, device=dev)

        # the expert weights are packed once, as at weight-load time
        eWp = mr.mr_expert_pack_weights(eW, stream=stream)

        def fused():
            mr.mr_expert_gemm_gather_packed(ex, we.k, eperm, eoff, eWp, we.N_r, n_out, out=eout,
                                            stream=stream)

        def fused_plain_layout():
            mr.mr_expert_gemm_gather(ex, we.k, eperm, eoff, eW, out=eout, stream=stream)

        def gemm_on_sorted_rows():
            mr.mr_expert_gemm_gather_packed(exs, we.k, None, eoff, eWp, we.N_r, n_out, out=eout,
                                            stream=stream)

        def unfused():
            mr.mr_gather_rows(ex, we.k, perm=eperm, inv_perm=einv, xs=exs, stream=stream)
            gemm_on_sorted_rows()

        # the combine fused into the same layer's epilogue (n_out-wide rows:
        # weighted sum over the k slots, shared add) beside the layer's
        # expert outputs written out and then mr_combine
        egen = torch.Generator(device=dev)
        egen.manual_seed(we.seed + 1)
        esh = torch.randn((we.T, n_out), generator=egen, device=dev).to(torch.bfloat16)
        eacc = torch.empty((we.T, n_out), dtype=torch.float32, device=dev)
        ey = torch.empty((we.T, n_out), dtype=torch.bfloat16, device=dev)

        def fused_combine():
            mr.mr_expert_gemm_gather_combine(ex, we.k, eperm, eoff, eWp, ewt, esh, N_r=we.N_r,
                                             n_out=n_out, packed=True, acc=eacc, y=ey,
                                             stream=stream)

        def layer_then_combine():
            fused()
            mr.mr_combine(eout, ewt, einv, esh, y=ey, stream=stream)

        fms = time_alone(fused, n_alone)
        pms = time_alone(fused_plain_layout, max(3, n_alone // 4))
        ums = time_alone(unfused, n_alone)
        gms = time_alone(gemm_on_sorted_rows, n_alone)
        cms = time_alone(fused_combine, n_alone)
        lcms = time_alone(layer_then_combine, n_alone)
        ef = 2.0 * we.T * we.k * we.d * n_out
        wbytes = 2 * we.N_r * n_out * we.d
        expert = {"workload": we.name, "n_out": n_out, "ms": fms,
                  "ms_with_combine_fused": cms,
                  "ms_layer_then_combine": lcms,
                  "combine_fused_note": "mr_expert_gemm_gather_combine (memset of the fp32 "
                                        "accumulator, GEMM with the weighted-sum epilogue, "
                                        "finalize with the shared add) against the layer's "
                                        "outputs written out and mr_combine",
                  "tflops": ef / (fms / 1e3) / 1e12,
                  "weights": "packed tiles (mr_expert_pack_weights, once, outside the timing)",
                  "ms_plain_weight_layout": pms,
                  "ms_unfused_gather_then_gemm": ums,
                  "ms_grouped_gemm_on_sorted_rows_alone": gms, "rows": we.T * we.k,
                  "expert_weight_bytes": wbytes,
                  "hbm_bound_ms": None,
                  "saved_bytes": 2 * 2 * we.T * we.k * we.d,
                  "l2": "read pass over 512 MB before each call"}
        del ex, ews, eW, eWp, eout, exs, esh, eacc, ey
        assert mr.mr_get_error(stream) == mr.MR_OK

    # Expert parallelism over peer memory, 8 ranks emulated on this GPU: each
    # rank routes a DeepSeek-V3 prefill batch of its own seed with the shared
    # gate, and every owner's receive buffer lives in this GPU's memory (with
    # 8 GPUs, the stores to the 7 other owners would cross NVLink instead).
    # Timed alone: one source's mr_ep_dispatch_p2p (destinations + its rows
    # stored into the 8 owners' buffers) beside mr_gather_rows of the same
    # rows into one buffer, and one source's mr_ep_combine_p2p reading the 8
    # buffers (identity experts) beside mr_combine of its own sorted rows.
    ep_stage = None
    if args.workload == wl.V3_FULL.name and not args.no_extra_stages:
        n_ep, wp = 8, wl.V3_PREFILL
        E_loc = wp.N_r // n_ep
        gate = wl.gen_router_inputs(wp)
        gW = torch.from_numpy(gate["W"]).to(dev)
        gb = torch.from_numpy(gate["b"]).to(dev)
        gws = torch.empty(max(4, mr.mr_router_workspace_size(wp.T, wp.d, wp.N_r)),
                          dtype=torch.uint8, device=dev)
        srcs = []
        for r in range(n_ep):
            xin = gate if r == 0 else wl.gen_router_inputs(wp.replace(seed=wp.seed + 7919 * r))
            rx = torch.from_numpy(xin["x_bf16"]).view(torch.bfloat16).to(dev)
            ridx, rwt = mr.mr_router_forward_ex(rx, gW, gb, wp.n_group, wp.topk_group, wp.k,
                                                wp.route_scale, wp.mask_mode,
                                                precision=mr.MR_PREC_BF16X3, workspace=gws,
                                                stream=stream)
            rc, ro, rperm, rinv = mr.mr_dispatch(ridx, wp.N_r, stream=stream)
            srcs.append(dict(x=rx, idx=ridx, w=rwt, counts=rc, offsets=ro, perm=rperm, inv=rinv))
        counts_all = torch.stack([s_["counts"] for s_ in srcs]).contiguous()
        per_owner = counts_all.cpu().numpy().reshape(n_ep, n_ep, E_loc).sum(axis=(0, 2))
        cap = int(per_owner.max())
        bufs = [torch.empty((cap, wp.d), dtype=torch.bfloat16, device=dev) for _ in range(n_ep)]
        for r, s_ in enumerate(srcs):  # every owner's buffer filled once
            s_["dest"], s_["lc"], s_["lo"] = mr.mr_ep_dispatch_p2p(
                s_["x"], s_["idx"], s_["inv"], s_["offsets"], counts_all, r, bufs, cap,
                stream=stream)
        s0 = srcs[0]
        xs0 = torch.empty((wp.T * wp.k, wp.d), dtype=torch.bfloat16, device=dev)
        sh0 = torch.randn((wp.T, wp.d), generator=torch.Generator(dev).manual_seed(wp.seed),
                          device=dev).to(torch.bfloat16)
        y0 = torch.empty((wp.T, wp.d), dtype=torch.bfloat16, device=dev)

        def p2p_dispatch():
            mr.mr_ep_dispatch_p2p(s0["x"], s0["idx"], s0["inv"], s0["offsets"], counts_all, 0,
                                  bufs, cap, dest=s0["dest"], local_counts=s0["lc"],
                                  local_offsets=s0["lo"], stream=stream)

        def local_gather():
            mr.mr_gather_rows(s0["x"], wp.k, perm=s0["perm"], inv_perm=s0["inv"], xs=xs0,
                              stream=stream)

        def p2p_combine():
            mr.mr_ep_combine_p2p(bufs, s0["w"], s0["idx"], s0["dest"], wp.N_r, cap, wp.d,
                                 torch.bfloat16, sh0, y=y0, stream=stream)

        def local_combine():
            mr.mr_combine(xs0, s0["w"], s0["inv"], sh0, y=y0, stream=stream)

        pd_ms = time_alone(p2p_dispatch, n_alone)
        lg_ms = time_alone(local_gather, n_alone)
        pc_ms = time_alone(p2p_combine, n_alone)
        lc_ms = time_alone(local_combine, n_alone)
        assert mr.mr_get_error(stream) == mr.MR_OK
        rows_b = wp.T * wp.k * wp.d * 2
        d_bytes = wp.T * wp.d * 2 + rows_b + 3 * 4 * wp.T * wp.k  # x, rows, idx/inv/dest
        c_bytes = rows_b + 2 * wp.T * wp.d * 2 + 3 * 4 * wp.T * wp.k  # rows, shared + y, w/idx/dest
        remote = int(((s0["idx"] // E_loc) != 0).sum().item())
        ep_stage = {
            "workload": f"{n_ep} ranks x {wp.name}, ranks emulated on one GPU "
                        "(every owner's buffer in this GPU's memory)",
            "capacity_rows": cap, "rows_per_source": wp.T * wp.k,
            "rows_to_other_owners": remote,
            "dispatch_p2p_ms": pd_ms, "dispatch_p2p_gbs": d_bytes / (pd_ms / 1e3) / 1e9,
            "gather_one_buffer_ms": lg_ms,
            "combine_p2p_ms": pc_ms, "combine_p2p_gbs": c_bytes / (pc_ms / 1e3) / 1e9,
            "combine_one_buffer_ms": lc_ms,
            "nvlink_bound_ms_8_gpus": remote * wp.d * 2 / (NVLINK_PEER_GBS * 1e9) * 1e3,
            "nvlink_note": f"rows to the other owners / {NVLINK_PEER_GBS} GB/s per direction "
                           "(B200 peer copy, measured; 900 nominal): the dispatch's bound "
                           "on 8 GPUs, unmeasured here",
            "l2": "read pass over 512 MB before each call"}
        del srcs, bufs, xs0, sh0, y0, gW, gb, gws, counts_all

    # The decode-size router (one position x batch 64): W read once per call.
    # Main figure: the plain entry point with the config's fp32 rows (split-K
    # over all SMs + reduce-and-route, no workspace).  Beside it: bf16 rows
    # through mr_router_forward_ex, a CUDA-graph replay, and the same call after
    # a write flush (dirty L2 lines) instead of a read pass.
    decode = None
    if args.workload == wl.V3_FULL.name:
        wd = wl.V3_DECODE
        dd_in = wl.gen_router_inputs(wd)
        dx32 = torch.from_numpy(dd_in["x_f32"]).to(dev)
        dx = torch.from_numpy(dd_in["x_bf16"]).view(torch.bfloat16).to(dev)
        dW = torch.from_numpy(dd_in["W"]).to(dev)
        db = torch.from_numpy(dd_in["b"]).to(dev)
        didx = torch.empty((wd.T, wd.k), dtype=torch.int32, device=dev)
        dwt = torch.empty((wd.T, wd.k), dtype=torch.float32, device=dev)
        dws = torch.empty(max(4, mr.mr_router_workspace_size(wd.T, wd.d, wd.N_r)),
                          dtype=torch.uint8, device=dev)

        def dplain():
            mr.mr_router_forward(dx32, dW, db, wd.n_group, wd.topk_group, wd.k, wd.route_scale,
                                 wd.mask_mode, idx_out=didx, w_out=dwt, stream=stream)

        def dbf16():
            mr.mr_router_forward_ex(dx, dW, db, wd.n_group, wd.topk_group, wd.k, wd.route_scale,
                                    wd.mask_mode, precision=mr.MR_PREC_BF16X3, idx_out=didx,
                                    w_out=dwt, workspace=dws, stream=stream)

        n_dec = 100
        l0 = mr.mr_launch_count()
        dplain()
        dlaunch = mr.mr_launch_count() - l0
        dus = time_alone(dplain, n_dec) * 1e3
        dus_mean = alone_means[dplain] * 1e3
        dus_write = time_alone(dplain, n_dec, write_flush) * 1e3

        # Per-call events resolve the call in coarse steps (≈ 2 us here), so
        # the call is also timed amortised: 200 x (read pass + call) minus
        # 200 x (read pass), two event pairs each, median of 5.
        def amortised(fn, n=200):
            def loop(with_fn):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(n):
                    read_flush()
                    if with_fn:
                        fn()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                return e0.elapsed_time(e1) * 1e3 / n
            loop(True)
            loop(False)
            return float(np.median([loop(True) - loop(False) for _ in range(5)]))

        dus_am = amortised(dplain)
        bus = time_alone(dbf16, n_dec) * 1e3
        gus, gerr = None, None
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                dplain()
            def replay():
                with torch.cuda.stream(stream):  # replay on the timed stream
                    graph.replay()

            gus = time_alone(replay, n_dec) * 1e3
            del graph
        except Exception as ex:  # report, do not fail the bench
            gerr = f"{type(ex).__name__}: {ex}"[:200]
        dbytes = 4 * wd.N_r * wd.d + 4 * wd.T * wd.d + 4 * wd.N_r + 8 * wd.T * wd.k
        bbytes = 4 * wd.N_r * wd.d + 2 * wd.T * wd.d + 4 * wd.N_r + 8 * wd.T * wd.k
        decode = {"workload": wd.name, "entry_point": "mr_router_forward (fp32 rows)",
                  "us": dus, "us_mean": dus_mean, "statistic": "median of 100 calls",
                  "us_amortised": dus_am,
                  "us_amortised_statistic": "(200 x (read pass + call) - 200 x read pass) / 200, "
                                            "median of 5",
                  "gbs_amortised": dbytes / (dus_am * 1e-6) / 1e9,
                  "launches_per_call": int(dlaunch),
                  "algorithmic_bytes": dbytes, "gbs": dbytes / (dus * 1e-6) / 1e9,
                  "us_cuda_graph": gus,
                  "gbs_cuda_graph": dbytes / (gus * 1e-6) / 1e9 if gus else None,
                  "us_after_write_flush": dus_write,
                  "us_bf16_rows_ex": bus,
                  "gbs_bf16_rows_ex": bbytes / (bus * 1e-6) / 1e9,
                  "l2": "read pass over 512 MB before every call (us_after_write_flush: "
                        "a 512 MB write instead)"}
        if gerr:
            decode["cuda_graph_error"] = gerr
        assert mr.mr_get_error(stream) == mr.MR_OK
    del flush, flush_i32

    # ---- end to end: pinned host inputs -> device -> path -> host result ----
    # Every step copies its inputs in from pinned host memory and its results
    # (y, idx, w) back out, all inside the timed region.  Three streams
    # (copies in, the path, copies out) and two sets of device buffers let
    # step i's results go out and step i+1's path run while step i+2's inputs
    # come in: PCIe carries the two directions at once, so the step costs
    # its host -> device bytes at the link's rate.
    e2e = None
    if not args.no_e2e:
        h_x = torch.empty_like(xb, device="cpu").pin_memory()
        h_E = torch.empty_like(E, device="cpu").pin_memory()
        h_sh = torch.empty_like(shared, device="cpu").pin_memory()
        h_y = torch.empty_like(y, device="cpu").pin_memory()
        h_idx = torch.empty_like(idx, device="cpu").pin_memory()
        h_w = torch.empty_like(wt, device="cpu").pin_memory()
        for h, g in ((h_x, xb), (h_E, E), (h_sh, shared)):
            h.copy_(g)
        h2d = sum(t.numel() * t.element_size() for t in (h_x, h_E, h_sh))
        d2h = sum(t.numel() * t.element_size() for t in (h_y, h_idx, h_w))
        sets = [main_set, {key: torch.empty_like(t) for key, t in main_set.items()}]
        s_in = torch.cuda.Stream(dev)
        s_out = torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in sets]    # inputs of the set landed
        ev_done = [torch.cuda.Event() for _ in sets]  # the path finished with the set
        ev_out = [torch.cuda.Event() for _ in sets]   # its results copied out

        def e2e_step(i):
            b = sets[i % 2]
            if i >= 2:
                s_in.wait_event(ev_done[i % 2])  # the path of step i-2 read this set
            with torch.cuda.stream(s_in):
                b["x"].copy_(h_x, non_blocking=True)
                b["E"].copy_(h_E, non_blocking=True)
                b["shared"].copy_(h_sh, non_blocking=True)
            ev_in[i % 2].record(s_in)
            stream.wait_event(ev_in[i % 2])
            if i >= 2:
                stream.wait_event(ev_out[i % 2])  # step i-2's results are out
            step(bufs=b)
            ev_done[i % 2].record(stream)
            s_out.wait_event(ev_done[i % 2])
            with torch.cuda.stream(s_out):
                h_y.copy_(b["y"], non_blocking=True)
                h_idx.copy_(b["idx"], non_blocking=True)
                h_w.copy_(b["wt"], non_blocking=True)
            ev_out[i % 2].record(s_out)

        n_e2e = max(2, min(args.steps, 10))
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        assert mr.mr_get_error(stream) == mr.MR_OK
        barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        s1.record(s_out)  # after the last step's results (s_out waited on all before)
        torch.cuda.synchronize(dev)
        e_ms = s0.elapsed_time(s1) / n_e2e
        assert mr.mr_get_error(stream) == mr.MR_OK
        e2e = {"value": aggregate_tokens_per_s(world, w.T, max_over_ranks(e_ms, world, dev)),
               "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e,
               "pipelining": "copies in, path and copies out on three streams over two "
                             "buffer sets; every step's copies inside the timed region"}
        del sets

    if rank != 0:
        return
    peaks = _peaks()
    T, dd, k, N = w.T, w.d, w.k, w.N_r
    rb = 2 if bf16_rows else 4                                 # row element bytes
    bytes_combine = T * (rb * k * dd + 2 * rb * dd + 8 * k)   # E rows, shared, y, w, inv
    bytes_gather = T * (rb * dd + rb * k * dd + 4 * k)        # x row once, k copies, inv
    bytes_router = T * (rb * dd + 8 * k) + 4 * N * dd + 4 * N  # x, idx/w, W, bias
    bytes_dispatch = T * k * (4 + 12)                         # idx in; perm, inv, ~scan out
    flops_router = 2.0 * T * dd * N
    comb_s = stage_ms["combine"] / 1e3
    # Roofline of the whole step: each stage's bound time at the measured
    # peaks (router: the slower of its bytes at HBM bandwidth and its
    # algorithmic flops at the bf16 tensor peak), summed, over the step time.
    hbm = peaks["hbm_gbs"] * 1e9
    bound_us = {"router": 1e6 * max(bytes_router / hbm, flops_router / (peaks["bf16_tflops"] * 1e12)),
                "dispatch": 1e6 * bytes_dispatch / hbm, "gather": 1e6 * bytes_gather / hbm,
                "combine": 1e6 * bytes_combine / hbm}
    achieved = bytes_combine / comb_s / 1e9
    traffic = None
    ent = NCU_TRAFFIC.get("combine")
    if ent and ent.get("src") == _src_sha("token_dispatch_fp32_b200/csrc/combine.cuh"):
        traffic = ent["bytes"]
    # Tensor work the router issues: three products per multiply-add, either
    # bf16 (bf16x3) or tf32 (3xTF32, tf32 peak = bf16 peak x 0.5 nominal).
    r_s = stage_ms["router"] / 1e3
    issue_peak = peaks["bf16_tflops"] * (1.0 if bf16_rows else 0.5)
    stages = {
        "router": {"ms": stage_ms["router"],
                   "arithmetic": "bf16x3 (bf16 rows, W in three bf16 planes, exact products, "
                                 "fp32 accumulation)" if bf16_rows else "3xTF32",
                   "ms_3xtf32_on_fp32_cast": alt_ms,
                   "tflops_algorithmic": flops_router / r_s / 1e12,
                   "tflops_issued": 3 * flops_router / r_s / 1e12,
                   "issue_peak_tflops": issue_peak,
                   "issue_peak_kind": "bf16 dense (measured)" if bf16_rows
                                      else "tf32 dense = 0.5 x measured bf16",
                   "frac_issued_of_peak": 3 * flops_router / r_s / 1e12 / issue_peak,
                   "frac_algorithmic_of_bf16_peak":
                       flops_router / r_s / 1e12 / peaks["bf16_tflops"],
                   "gbs": bytes_router / r_s / 1e9},
        "dispatch": {"ms": stage_ms["dispatch"],
                     "gbs": bytes_dispatch / (stage_ms["dispatch"] / 1e3) / 1e9},
        "gather": {"ms": stage_ms["gather"],
                   "gbs": bytes_gather / (stage_ms["gather"] / 1e3) / 1e9,
                   "frac_hbm": bytes_gather / (stage_ms["gather"] / 1e3) / 1e9 / peaks["hbm_gbs"]},
        "combine": {"ms": stage_ms["combine"], "gbs": achieved,
                    "frac_hbm": achieved / peaks["hbm_gbs"]},
    }
    tf32_peak = 0.5 * peaks["bf16_tflops"]
    if alt_ms is not None:
        stages["router_3xtf32_fp32_rows"] = {
            "ms": alt_ms, "tflops_issued": 3 * flops_router / (alt_ms / 1e3) / 1e12,
            "issue_peak_tflops": tf32_peak, "issue_peak_kind": "tf32 dense = 0.5 x bf16",
            "frac_issued_of_peak": 3 * flops_router / (alt_ms / 1e3) / 1e12 / tf32_peak}
    if tf32_ms is not None:
        stages["router_tf32_fp32_rows"] = {
            "ms": tf32_ms, "arithmetic": "plain TF32: one tf32 product per multiply-add, "
                                         "fp32 accumulation (logits within ~1e-3 relative)",
            "tflops": flops_router / (tf32_ms / 1e3) / 1e12, "peak_tflops": tf32_peak,
            "peak_kind": "tf32 dense = 0.5 x bf16",
            "frac_of_peak": flops_router / (tf32_ms / 1e3) / 1e12 / tf32_peak}
    for key, st in other_routers.items():
        st["frac_issued_of_bf16_peak"] = st["tflops_issued"] / peaks["bf16_tflops"]
        st["frac_algorithmic_of_bf16_peak"] = st["tflops_algorithmic"] / peaks["bf16_tflops"]
        stages[key] = st
    if expert is not None:
        expert["frac_of_bf16_peak"] = expert["tflops"] / peaks["bf16_tflops"]
        # every expert's weights read once from HBM, against the tensor time
        expert["hbm_bound_ms"] = expert["expert_weight_bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e3
        expert["roofline_ms"] = max(expert["hbm_bound_ms"], 2.0 * expert["rows"] * 7168 *
                                    expert["n_out"] / (peaks["bf16_tflops"] * 1e12) * 1e3)
        expert["frac_of_roofline"] = expert["roofline_ms"] / expert["ms"]
        stages["expert_gemm_gather_deepseek_v3_prefill_T4096"] = expert
    if ep_stage is not None:
        ep_stage["dispatch_p2p_frac_hbm"] = ep_stage["dispatch_p2p_gbs"] / peaks["hbm_gbs"]
        ep_stage["combine_p2p_frac_hbm"] = ep_stage["combine_p2p_gbs"] / peaks["hbm_gbs"]
        stages["ep_p2p_deepseek_v3_prefill_8_ranks"] = ep_stage
    if decode is not None:
        decode["frac_hbm"] = decode["gbs"] / peaks["hbm_gbs"]
        if decode.get("gbs_cuda_graph"):
            decode["frac_hbm_cuda_graph"] = decode["gbs_cuda_graph"] / peaks["hbm_gbs"]
        stages["decode_router"] = decode
    line = {
        "metric": METRIC, "value": aggregate_tokens_per_s(world, T, ms_max), "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; x/W/b numpy PCG64, expert outputs and shared output "
                "torch Philox on device)",
        "config": _config(w),
        "roofline": {"bound": "hbm", "kernel": "combine", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": traffic, "algorithmic_bytes": bytes_combine,
                     "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)"
                     if peaks["source"] == "measured" else "fallback 6650 GB/s",
                     "step_frac": sum(bound_us.values()) / (ms_max * 1e3),
                     "step_bound_us": bound_us,
                     "step_frac_note": "sum of the stages' roofline times at the measured "
                                       "peaks (router: max of HBM bytes and algorithmic flops "
                                       "at the bf16 peak) / ms_per_step"},
        "stages": stages,
        "gpu_launches": int(launches),
        "clocks": clk,
        "e2e": e2e,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, gpu_router=step_router_out)
        line["near_ties"] = line["cpu_baseline"].pop("router_check")
    print(json.dumps(line), flush=True)


def _free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _spawned_rank(rank: int, argv, world: int, port: int):
    """Entry of a rank started by spawn_ranks: the launcher's environment
    (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR, MASTER_PORT), then main()."""
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    main(argv)


def spawn_ranks(argv, world: int):
    """`--gpus N` without a launcher: start N ranks here (one process per
    GPU, spawn start method), each with the environment torchrun would give
    it, and wait for them; a failing rank fails the run."""
    import torch.multiprocessing as tmp
    tmp.start_processes(_spawned_rank, args=(argv, world, _free_port()), nprocs=world,
                        join=True, start_method="spawn")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=wl.V3_FULL.name, choices=[x.name for x in wl.ALL])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-stages", action="store_true",
                    help="skip the prefill-router stages timed beside the step")
    ap.add_argument("--expert-weights", choices=("packed", "plain"), default="packed",
                    help="with --only expert: the expert weights' layout")
    ap.add_argument("--expert-rows", choices=("gathered", "sorted"), default="gathered",
                    help="with --only expert: rows gathered in the GEMM, or pre-sorted")
    ap.add_argument("--n-out", type=int, default=2048,
                    help="with --only expert: output columns of the expert layer")
    ap.add_argument("--only", choices=("router", "expert"), default=None,
                    help="time one stage alone (a profiling aid; no bench line)")
    ap.add_argument("--expert-epilogue", choices=("out", "combine"), default="out",
                    help="with --only expert: write the expert outputs, or fuse the weighted "
                         "combine and shared add (mr_expert_gemm_gather_combine)")
    ap.add_argument("--router-weights", choices=("f32", "bf16"), default="f32",
                    help="with --only router: the gate weight's stored type")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    w = wl.BY_NAME[args.workload]
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        spawn_ranks(sys.argv[1:] if argv is None else argv, args.gpus)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU "
              f"(torchrun --nproc-per-node {args.gpus}) or drop the launcher", file=sys.stderr)
        sys.exit(2)
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if args.only == "router":
        run_router_only(args, w)
        return
    if args.only == "expert":
        run_expert_only(args, w)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, w, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
