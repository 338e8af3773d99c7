"""Benchmark of the Sol-Attn hot path on B200: QK-RMSNorm + 3D RoPE ->
block select -> block-sparse attention, one pass of the whole chain per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--impl ours|reference]
                    [--chain fused|split]

The default step is the fused chain: the prologue also emits the block means
(sol_qk_prologue_pool), the selection scores them (sol_block_select_pooled),
then attention; the split chain (sol_qk_prologue, sol_block_select, which pools
q and k itself) is timed afterwards for comparison and reported beside it.

Prints ONE JSON line (rank 0).  `value` is the selected-FLOP rate of the whole
chain step (selected attention FLOPs / device time of prologue + select +
attention), summed over ranks; each rank runs its own independent clip of the
workload (weak scaling, no collective on the data path).  Inputs stay resident
in HBM during the device-timed region and are far larger than L2 (no flush
needed).  `e2e` times the same chain through host buffers: pinned host -> device
copies of the raw Q, K, V and the device -> host copy of O and LSE are inside
the timed region.  `--impl reference` times the fp64 CPU oracle on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FP32_LANES = 148 * 128                # fp32 FMA lanes of a B200 (148 SMs x 128)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


KERNEL_SOURCES = ("block_sparse_attention_sol_b200/csrc/attn_sm100.cuh",
                  "block_sparse_attention_sol_b200/csrc/sm100_ptx.cuh",
                  "block_sparse_attention_sol_b200/csrc/blocks.cuh")


def load_ncu_traffic(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None
    when there is none or the kernel sources changed since it was measured."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for src in KERNEL_SOURCES:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                key, val = line.split(":", 1)
                fields[key.strip()] = val.strip()
    if fields.get("kernel_source_sha256") != h.hexdigest():
        return None
    return float(fields["dram_bytes_per_launch"])


def kernel_sources_sha256() -> str:
    """Hash of the CUDA sources and the C header, the stamp the GPU parity tests put on their record."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_sol_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    with open(os.path.join(ROOT, "include", "sol.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def load_parity():
    """The GPU parity tests' record (tests/parity_record.json): per workload and path,
    selection rows compared with the oracle, near-tie rows, differing rows and the
    attention errors; flagged stale when the kernel sources changed since."""
    path = os.path.join(ROOT, "tests", "parity_record.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    cur = kernel_sources_sha256()
    keep = ("rows", "near_tie_rows", "differing_rows", "attention_units", "max_abs_dO", "max_abs_dLSE")
    out = {"record": "tests/parity_record.json", "rule": "ids bit-exact outside near-tie rows (oracle k-th and "
           "(k+1)-th scores closer than 1e-4 relative); |dO| <= 2e-2, |dLSE| <= 1e-2",
           "kernel_sources_match": all(e.get("kernel_sources_sha256") == cur for e in rec.get("entries", {}).values()),
           "workloads": {}}
    for key, e in rec.get("entries", {}).items():
        wl_name, path_name = key.split("/", 1)
        out["workloads"].setdefault(wl_name, {})[path_name] = {k: e[k] for k in keep if k in e}
    return out


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.device = device

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            cmd += ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except FileNotFoundError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- oracle timing
def oracle_attention_sample(wl, inp, topk, n_units: int, seed: int):
    """Times the fp64 oracle on n_units (b, h, query block) units of the workload
    with random valid selections; returns (selected FLOPs, seconds, threads)."""
    import oracle as orc
    from workloads import random_index_lists
    rng = np.random.default_rng([seed, 17])
    q, k, v = (inp[n].float().numpy() for n in ("q", "k", "v"))
    idx = random_index_lists(1, 1, wl.nb, topk, seed=seed).numpy()[0, 0]
    flops = 0
    t0 = time.perf_counter()
    for _ in range(n_units):
        b, h, i = int(rng.integers(0, wl.B)), int(rng.integers(0, wl.H)), int(rng.integers(0, wl.nb))
        sel = np.zeros((wl.B, wl.H, wl.nb, topk), dtype=np.int32)
        sel[b, h, i] = idx[i]
        orc.sparse_attention_rows(q, k, v, sel, wl.block, 1.0 / math.sqrt(wl.D), b, h, i)
        nq = min(wl.block, wl.N - i * wl.block)
        nk = sum(min(wl.block, wl.N - j * wl.block) for j in idx[i])
        flops += 4 * nq * nk * wl.D
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        threads = 1
    return flops, dt, threads


def oracle_prep_sample(wl, inp, topk, n_tokens: int = 1024):
    """Times the fp64 oracle's prologue on n_tokens tokens of Q and K, and its
    selection (block means, all scores, top-k) on the whole workload; returns
    (prologue GB/s, prologue s, select GB/s, select s) over the bytes the GPU
    stages move (prologue: read raw q, k and write q, k as bf16; selection: read
    q, k as bf16 and write the ids)."""
    import oracle as orc
    q32, k32 = inp["q"].float().numpy(), inp["k"].float().numpy()
    gq, gk = inp["gamma_q"].double().numpy(), inp["gamma_k"].double().numpy()
    rng = np.random.default_rng(11)
    tok = np.sort(rng.choice(wl.N, size=min(n_tokens, wl.N), replace=False))
    t0 = time.perf_counter()
    orc.qk_prologue(q32, gq, wl.grid, wl.rope_split, wl.rope_theta, wl.eps, tokens=tok)
    orc.qk_prologue(k32, gk, wl.grid, wl.rope_split, wl.rope_theta, wl.eps, tokens=tok)
    t_pro = time.perf_counter() - t0
    pro_bytes = 4 * wl.B * len(tok) * wl.H * wl.D * 2
    t0 = time.perf_counter()
    orc.block_select(q32, k32, wl.block, topk)
    t_sel = time.perf_counter() - t0
    sel_bytes = 2 * wl.B * wl.N * wl.H * wl.D * 2 + 4 * wl.B * wl.H * wl.nb * topk
    return pro_bytes / t_pro / 1e9, t_pro, len(tok), sel_bytes / t_sel / 1e9, t_sel


def time_workload(sol, wl, dev, stream, seed, steps: int, warmup: int, peaks):
    """The fused chain on another workload (per-stage CUDA-event times over
    `steps` steps after `warmup`); the selected FLOPs are counted from the ids
    the step produced (exact for a short last block)."""
    topk = wl.topk[0]
    inp = make_inputs(wl, seed=seed)
    d = {n: inp[n].to(dev) for n in ("q", "k", "v", "gamma_q", "gamma_k")}
    del inp
    q, k, o = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["q"])
    lse = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.B, wl.H, wl.nb, topk), dtype=torch.int32, device=dev)
    qbar = torch.empty((wl.B, wl.H, wl.nb, wl.D), dtype=torch.float32, device=dev)
    kbar = torch.empty_like(qbar)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        sol.sol_qk_prologue_pool(d["q"], d["k"], d["gamma_q"], d["gamma_k"], wl.grid, wl.block, wl.rope_split,
                                 wl.rope_theta, wl.eps, q_out=q, k_out=k, qbar_out=qbar, kbar_out=kbar)
        if ev is not None:
            ev[1].record(stream)
        sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, topk, idx_out=idx)
        if ev is not None:
            ev[2].record(stream)
        sol.sol_sparse_attn_fwd(q, k, d["v"], idx, wl.grid, wl.block, o=o, lse=lse)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(warmup):
        step()
    for s_ in range(steps):
        step(evs[s_])
    torch.cuda.synchronize(dev)
    if sol.sol_check_device_status() != sol.SOL_OK:
        raise RuntimeError(f"device-side error on workload {wl.config_id}")
    st = {name: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / steps
          for i, name in enumerate(("prologue", "select", "attention"))}
    sizes = torch.clamp(wl.N - torch.arange(wl.nb, device=dev) * wl.block, max=wl.block).to(torch.float64)
    flops = float(4 * wl.D * (sizes[idx.long()].sum(-1) * sizes).sum().item())
    io = wl.B * wl.N * wl.H * wl.D * 2
    pooled = 2 * wl.B * wl.H * wl.nb * wl.D * 4
    idx_b = 4 * wl.B * wl.H * wl.nb * topk
    pro_b, prep_b = 4 * io + pooled, 4 * io + idx_b
    return {"workload": wl.name, "config_id": wl.config_id, "N": wl.N, "topk": topk,
            "selected_tflop": flops / 1e12, "steps": steps,
            "attention": {"ms": st["attention"], "TFLOP/s": flops / st["attention"] / 1e9,
                          "frac_bf16_burst": flops / st["attention"] / 1e9 / peaks["bf16_tflops"]},
            "prologue": {"ms": st["prologue"], "GB/s": pro_b / st["prologue"] / 1e6,
                         "frac_hbm": pro_b / st["prologue"] / 1e6 / peaks["hbm_gbs"]},
            "select": {"ms": st["select"], "scoring_TFLOP/s_fp32": 2 * wl.B * wl.H * wl.nb * wl.nb * wl.D /
                       st["select"] / 1e9},
            "preparation": {"ms": st["prologue"] + st["select"],
                            "frac_hbm": prep_b / (st["prologue"] + st["select"]) / 1e6 / peaks["hbm_gbs"]},
            "chain_ms": sum(st.values()), "chain_TFLOP/s": flops / sum(st.values()) / 1e9}


def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    topk = wl.topk[0]
    inp = make_inputs(wl, seed=0, names=("q", "k", "v"))
    units = args.ref_units
    for _ in range(args.warmup):
        oracle_attention_sample(wl, inp, topk, 1, seed=123)
    tot_f, tot_t, threads = 0, 0.0, 1
    for s in range(args.steps):
        f, t, threads = oracle_attention_sample(wl, inp, topk, units, seed=s)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    sample = (f"fp64 oracle attention on {units} random (b, h, query block) units per step with k={topk} "
              f"random kept blocks of workload {wl.config_id}; value = their selected FLOPs / CPU time")
    line = {
        "impl": "reference", "metric": "sparse-attn effective TFLOP/s (selected FLOPs)", "value": value,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "config_id": wl.config_id, "B": wl.B, "N": wl.N, "H": wl.H, "D": wl.D,
                   "block": wl.block, "topk": topk, "parallelism": f"independent clip per rank x{world}"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
def run_ours(args, wl, world, rank, local):
    import block_sparse_attention_sol_b200 as sol
    topk = wl.topk[0]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    inp = make_inputs(wl, seed=rank)
    host = {n: inp[n].pin_memory() for n in ("q", "k", "v")}
    d = {n: inp[n].to(dev) for n in ("q", "k", "v", "gamma_q", "gamma_k")}
    q = torch.empty_like(d["q"])
    k = torch.empty_like(d["k"])
    o = torch.empty_like(d["q"])
    lse = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.B, wl.H, wl.nb, topk), dtype=torch.int32, device=dev)
    shape = sol.SolShape(wl.B, wl.N, wl.H, wl.D, *wl.grid)
    ws = torch.empty(sol.sol_block_select_workspace_bytes(shape, wl.block), dtype=torch.uint8, device=dev)
    qbar = torch.empty((wl.B, wl.H, wl.nb, wl.D), dtype=torch.float32, device=dev)
    kbar = torch.empty_like(qbar)
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

    def chain(ev=None, fused=None):
        """One step of the hot path.  fused: prologue + block means in one pass, then
        the selection from the means (3 launches); else prologue, then the selection
        pooling from q and k itself (4 launches)."""
        fused = (args.chain == "fused") if fused is None else fused
        if ev is not None:
            ev[0].record(stream)
        if fused:
            sol.sol_qk_prologue_pool(d["q"], d["k"], d["gamma_q"], d["gamma_k"], wl.grid, wl.block, wl.rope_split,
                                     wl.rope_theta, wl.eps, q_out=q, k_out=k, qbar_out=qbar, kbar_out=kbar)
        else:
            sol.sol_qk_prologue(d["q"], d["k"], d["gamma_q"], d["gamma_k"], wl.grid, wl.rope_split, wl.rope_theta,
                                wl.eps, q_out=q, k_out=k)
        if ev is not None:
            ev[1].record(stream)
        if fused:
            sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, topk, idx_out=idx)
        else:
            sol.sol_block_select(q, k, wl.grid, wl.block, topk, workspace=ws, idx_out=idx)
        if ev is not None:
            ev[2].record(stream)
        sol.sol_sparse_attn_fwd(q, k, d["v"], idx, wl.grid, wl.block, o=o, lse=lse)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        chain()
    torch.cuda.synchronize(dev)
    if sol.sol_check_device_status() != sol.SOL_OK:
        raise RuntimeError("device-side error during warm-up")

    # device-timed region: inputs resident in HBM
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        barrier(world)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for s in range(args.steps):
            chain(evs[s])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    status = sol.sol_check_device_status()
    if status != sol.SOL_OK:
        raise RuntimeError(f"device-side error in the timed region: {sol.sol_status_string(status)}")
    ms_local = start.elapsed_time(stop) / args.steps
    ms = max_over_ranks(ms_local, world)
    stage_ms = {name: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps
                for i, name in enumerate(("prologue", "select", "attention"))}

    # the other chain variant, for comparison (not part of `value`)
    alt_steps = min(args.steps, 10)
    alt_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(alt_steps)]
    alt_fused = args.chain != "fused"
    chain(fused=alt_fused)
    for s_ in range(alt_steps):
        chain(alt_evs[s_], fused=alt_fused)
    torch.cuda.synchronize(dev)
    alt_ms = {name: sum(e[i].elapsed_time(e[i + 1]) for e in alt_evs) / alt_steps
              for i, name in enumerate(("prologue", "select", "attention"))}

    # FP8 (e4m3) variant of the attention on the same prologue outputs and selection,
    # for comparison (not part of `value`: reduced precision).  Its peak is the
    # measured bf16 rate x 2, the nominal e4m3 / bf16 ratio of the tensor cores.
    fp8 = None
    if not args.no_fp8:
        fin = sol.sol_quant_attn_fp8(q, k, d["v"], wl.grid)
        o8 = torch.empty_like(o)
        lse8 = torch.empty_like(lse)
        fp8_steps = min(args.steps, 10)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        sol.sol_sparse_attn_fwd_fp8(fin, idx, wl.grid, wl.block, o=o8, lse=lse8)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(fp8_steps):
            sol.sol_quant_attn_fp8(q, k, d["v"], wl.grid, out=fin)
        e1.record(stream)
        for _ in range(fp8_steps):
            sol.sol_sparse_attn_fwd_fp8(fin, idx, wl.grid, wl.block, o=o8, lse=lse8)
        e2.record(stream)
        torch.cuda.synchronize(dev)
        qms = e0.elapsed_time(e1) / fp8_steps
        ams = e1.elapsed_time(e2) / fp8_steps
        io_b = wl.B * wl.N * wl.H * wl.D * 2
        # read q, k once and v twice (its per-head max, then its codes); write three
        # e4m3 code tensors and the q, k row scales
        qbytes = 4 * io_b + 3 * io_b // 2 + 2 * 4 * wl.B * wl.H * wl.N
        fp8 = {"quantise_ms": qms, "quantise_GB/s": qbytes / qms / 1e6,
               "attention_ms": ams, "attention_TFLOP/s": wl.selected_flops(topk) / ams / 1e9}
    # Selection variants and tile blocks (opt-in, not part of `value`): each timed over
    # a few launches after one untimed launch, on the same prologue outputs.
    variants = None
    if args.variants:
        variants = {}
        nrep = min(args.steps, 10)

        def timed(fn):
            fn()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            a_.record(stream)
            for _ in range(nrep):
                out_ = fn()
            b_.record(stream)
            torch.cuda.synchronize(dev)
            return a_.elapsed_time(b_) / nrep, out_

        ms_plain, _ = timed(lambda: sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, topk, idx_out=idx))
        ms_forced, _ = timed(lambda: sol.sol_block_select_pooled_ex(qbar, kbar, wl.grid, wl.block, topk, flags=3))
        ms_topp, (idx_p, cnt_p) = timed(lambda: sol.sol_block_select_pooled_ex(qbar, kbar, wl.grid, wl.block, topk,
                                                                               flags=4, top_p=0.9, softmax_scale=2.0))
        ms_cnt, _ = timed(lambda: sol.sol_sparse_attn_fwd_counts(q, k, d["v"], idx_p, cnt_p, wl.grid, wl.block,
                                                                 o=o, lse=lse))
        kept = int(cnt_p.sum().item())
        flops_cnt = 4 * wl.block * wl.block * wl.D * kept          # every block of this workload is full
        variants["select_ms"] = {"plain": ms_plain, "forced_diagonal_first_frame": ms_forced,
                                 "top_p_0.9_scale_2": ms_topp}
        variants["attention_top_p_counts"] = {"ms": ms_cnt, "mean_count": kept / cnt_p.numel(),
                                              "TFLOP/s": flops_cnt / ms_cnt / 1e9}
        tile = (4, 4, 8) if wl.grid[0] % 4 == 0 and wl.grid[1] % 4 == 0 and wl.grid[2] % 8 == 0 else None
        if tile is not None:
            ms_tp, (qt, kt_, qbt, kbt) = timed(lambda: sol.sol_qk_prologue_pool_tiled(
                d["q"], d["k"], d["gamma_q"], d["gamma_k"], wl.grid, tile, wl.rope_split, wl.rope_theta, wl.eps,
                q_out=q, k_out=k))
            idx_t = sol.sol_block_select_pooled(qbt, kbt, wl.grid, wl.block, topk)
            ms_ta, _ = timed(lambda: sol.sol_sparse_attn_fwd_tiled(q, k, d["v"], idx_t, wl.grid, tile, o=o, lse=lse))
            variants["tiles_4x4x8"] = {"prologue_pool_ms": ms_tp, "attention_ms": ms_ta,
                                       "attention_TFLOP/s": wl.selected_flops(topk) / ms_ta / 1e9}
        if sol.sol_check_device_status() != sol.SOL_OK:
            raise RuntimeError("device-side error in the variant runs")
    # Backward pass (opt-in, not part of `value`): CUDA-core kernels, fp32 arithmetic.
    # FLOPs counted as 2.5 x the forward's selected FLOPs (five products against two).
    backward = None
    if args.backward:
        dout = torch.randn(o.shape, device=dev, dtype=torch.float32).to(o.dtype)
        sol.sol_sparse_attn_fwd(q, k, d["v"], idx, wl.grid, wl.block, o=o, lse=lse)
        ws_b = torch.empty(max(int(sol.lib.sol_sparse_attn_bwd_workspace_bytes(shape, wl.block)), 16),
                           dtype=torch.uint8, device=dev)
        sol.sol_sparse_attn_bwd(q, k, d["v"], o, lse, dout, idx, wl.grid, wl.block, workspace=ws_b)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        b0.record(stream)
        sol.sol_sparse_attn_bwd(q, k, d["v"], o, lse, dout, idx, wl.grid, wl.block, workspace=ws_b)
        b1.record(stream)
        torch.cuda.synchronize(dev)
        bms = b0.elapsed_time(b1)
        backward = {"ms": bms, "TFLOP/s": 2.5 * wl.selected_flops(topk) / bms / 1e9,
                    "kernels": "sol::attnbwd (CUDA cores, fp32)"}
    # End to end through host buffers, the way a caller streams clips: the pipeline
    # copies each step's raw Q, K, V in from pinned host memory, runs the fused chain
    # and copies O and LSE back, with the next step's inputs crossing PCIe while the
    # current step computes (double-buffered device buffers, three streams).
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v"))
    d2h = o_host.numel() * o_host.element_size() + lse_host.numel() * lse_host.element_size()
    e2e_ms = e2e_serial_ms = None
    if not args.no_e2e:
        from block_sparse_attention_sol_b200.pipeline import HostChainPipeline
        e2e_steps = args.e2e_steps or args.steps
        pipe = HostChainPipeline(wl.B, wl.N, wl.H, wl.D, wl.grid, wl.block, topk, d["gamma_q"], d["gamma_k"],
                                 dtype=d["q"].dtype, rope_split=wl.rope_split, rope_theta=wl.rope_theta, eps=wl.eps,
                                 device=dev)
        for _ in range(2):
            pipe.submit(host["q"], host["k"], host["v"], o_host, lse_host)
        pipe.synchronize()
        e2e_start, e2e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        e2e_start.record(pipe.s_in)
        for _ in range(e2e_steps):
            pipe.submit(host["q"], host["k"], host["v"], o_host, lse_host)
        e2e_stop.record(pipe.s_out)          # after the last copy-out, which follows every other step's work
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks(e2e_start.elapsed_time(e2e_stop) / e2e_steps, world)
        del pipe
        # the same through one stream, one step after another (for comparison)
        serial_steps = 3
        barrier(world)
        torch.cuda.synchronize(dev)
        e2e_start.record(stream)
        for _ in range(serial_steps):
            d["q"].copy_(host["q"], non_blocking=True)
            d["k"].copy_(host["k"], non_blocking=True)
            d["v"].copy_(host["v"], non_blocking=True)
            chain()
            o_host.copy_(o, non_blocking=True)
            lse_host.copy_(lse, non_blocking=True)
        e2e_stop.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_serial_ms = max_over_ranks(e2e_start.elapsed_time(e2e_stop) / serial_steps, world)
    if sol.sol_check_device_status() != sol.SOL_OK:
        raise RuntimeError("device-side error in the end-to-end runs")

    flops = wl.selected_flops(topk)          # selected attention FLOPs of one step (one clip)
    value = flops * world / (ms * 1e-3) / 1e12
    e2e_value = None if e2e_ms is None else flops * world / (e2e_ms * 1e-3) / 1e12
    peaks = load_peaks()
    att_s = stage_ms["attention"] * 1e-3
    achieved = flops / att_s / 1e12
    # Peak: the measured burst bf16 GEMM rate.  The attention runs in a loop of
    # chain steps lasting about a second, far shorter than the seconds-long loop
    # the sustained figure comes from (measured at a much lower SM clock), so the
    # burst figure is the fair denominator; the sustained fraction is reported beside it.
    peak = peaks["bf16_tflops"]
    peak_sustained = peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]
    loop_s = ms * args.steps * 1e-3
    traffic = load_ncu_traffic("sparse_attn_fwd")
    io_bytes = wl.B * wl.N * wl.H * wl.D * 2
    idx_bytes = 4 * wl.B * wl.H * wl.nb * topk
    pooled_bytes = 2 * wl.B * wl.H * wl.nb * wl.D * 4
    score_flops = 2 * wl.B * wl.H * wl.nb * wl.nb * wl.D

    if fp8 is not None:
        fp8["peak_tflops_e4m3"] = 2 * peaks["bf16_tflops"]
        fp8["frac_e4m3_burst"] = fp8["attention_TFLOP/s"] / fp8["peak_tflops_e4m3"]
        fp8["frac_e4m3_sustained"] = fp8["attention_TFLOP/s"] / (2 * peak_sustained)
        fp8["quantise_frac_hbm"] = fp8["quantise_GB/s"] / peaks["hbm_gbs"]
        fp8["kernel"] = "sol::attnfp8::sparse_attn_fp8_kernel"

    clock_mhz = sampler.summary().get("sm_mhz") or 1965.0

    def stages(st, fused):
        """Per-stage rates.  Algorithmic bytes: prologue reads q_raw, k_raw and writes
        q, k (+ the block means when fused); the split selection reads q, k and writes
        idx, the fused one reads the means and writes idx.  `preparation` is prologue +
        selection against the bytes the pair must move (read q_raw, k_raw, write q, k, idx)."""
        pro_b = 4 * io_bytes + (pooled_bytes if fused else 0)
        sel_b = (pooled_bytes if fused else 2 * io_bytes) + idx_bytes
        prep_ms = st["prologue"] + st["select"]
        return {
            "chain": "fused" if fused else "split",
            "prologue": {"ms": st["prologue"], "GB/s": pro_b / st["prologue"] / 1e6,
                         "frac_hbm": pro_b / st["prologue"] / 1e6 / peaks["hbm_gbs"]},
            "select": {"ms": st["select"], "GB/s": sel_b / st["select"] / 1e6,
                       "frac_hbm": sel_b / st["select"] / 1e6 / peaks["hbm_gbs"],
                       "scoring_TFLOP/s_fp32": score_flops / st["select"] / 1e9,
                       # the selection moves little and computes much: its roofline is the fp32
                       # FMA rate, 148 SMs x 128 lanes x 2 FLOP at the sampled SM clock
                       "bound": "alu", "fp32_peak_tflops": FP32_LANES * 2 * clock_mhz * 1e-6,
                       "frac_fp32": score_flops / st["select"] / 1e9 / (FP32_LANES * 2 * clock_mhz * 1e-6)},
            "preparation": {"ms": prep_ms, "GB/s": (4 * io_bytes + idx_bytes) / prep_ms / 1e6,
                            "frac_hbm": (4 * io_bytes + idx_bytes) / prep_ms / 1e6 / peaks["hbm_gbs"]},
            "attention": {"ms": st["attention"], "TFLOP/s": flops / st["attention"] / 1e9,
                          "frac_bf16_burst": flops / st["attention"] / 1e9 / peak,
                          "frac_bf16_sustained": flops / st["attention"] / 1e9 / peak_sustained},
            "hbm_peak_gbs": peaks["hbm_gbs"],
        }
    clocks = sampler.summary()
    if rank != 0:
        return
    line = {
        "metric": "sparse-attn effective TFLOP/s (selected FLOPs)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "config_id": wl.config_id, "B": wl.B, "N": wl.N, "H": wl.H, "D": wl.D,
                   "grid": list(wl.grid), "block": wl.block, "topk": topk,
                   "selected_tflop_per_step": flops / 1e12,
                   "parallelism": f"independent clip per rank x{world}",
                   "l2": f"inputs {5 * io_bytes / 1e9:.1f} GB resident, > {L2_BYTES >> 20} MB L2; no flush"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "sol::attn100::sparse_attn_fwd_kernel",
                     "peak_source": f"{peaks['source']} bf16 dense GEMM, burst (the kernel is timed inside a "
                                    f"{loop_s:.1f} s loop of chain steps)",
                     "peak_sustained": peak_sustained, "frac_sustained": achieved / peak_sustained},
        "stages": stages(stage_ms, args.chain == "fused"),
        "stages_" + ("split" if args.chain == "fused" else "fused"): stages(alt_ms, args.chain != "fused"),
        "e2e": None if e2e_ms is None else {
            "value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_ms, "api": "block_sparse_attention_sol_b200.pipeline.HostChainPipeline",
            "overlap": "double-buffered over clips: step i+1's inputs cross PCIe while step i computes",
            "serial_ms_per_step": e2e_serial_ms},
        "fp8_attention": fp8,
        "variants": variants,
        "backward": backward,
        "gpu_launches": (3 if args.chain == "fused" else 4) * args.steps,
        "clocks": clocks,
    }
    line["parity"] = load_parity()
    if world == 1 and not args.no_cpu_baseline:
        f, t, threads = oracle_attention_sample(wl, inp, topk, args.cpu_units, seed=99)
        pro_gbs, pro_t, pro_tok, sel_gbs, sel_t = oracle_prep_sample(wl, inp, topk)
        line["cpu_baseline"] = {
            "value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle attention on {args.cpu_units} random (b, h, query block) units with "
                      f"k={topk} random kept blocks ({f / 1e9:.1f} GFLOP, {t:.1f} s)",
            "prologue": {"GB/s": pro_gbs, "s": pro_t,
                         "sample": f"fp64 oracle prologue of Q and K on {pro_tok} random tokens x {wl.H} heads; "
                                   f"GB/s over the bf16 bytes the GPU prologue moves for them"},
            "select": {"GB/s": sel_gbs, "s": sel_t,
                       "sample": "fp64 oracle block means, scores and top-k over the whole workload; GB/s over "
                                 "the bytes the GPU selection moves (read q, k as bf16, write the ids)"}}
    if world == 1 and not args.no_per_config:
        # the other bf16 workloads, fused chain, timed after everything above (not part of `value`)
        del d, q, k, o, lse, idx, qbar, kbar, ws, host, o_host, lse_host
        torch.cuda.empty_cache()
        line["per_config"] = [time_workload(sol, WORKLOADS[c], dev, stream, rank, args.per_config_steps, 3,
                                            load_peaks()) for c in (1, 2, 3) if c != wl.config_id]
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- sequence-parallel arm (opt-in)
def run_seqpar(args, wl, world, rank, local):
    """One clip over `world` ranks: each rank holds a token shard, the attention runs on
    head shards behind an INT8 Q/K/V and FP8 O all-to-all (strong scaling).  With one
    rank the exchange is a local copy and the line measures the quantisation kernels
    and the chain on quantised inputs."""
    import block_sparse_attention_sol_b200 as sol  # noqa: F401  (loads libsol)
    from block_sparse_attention_sol_b200.seqpar import CollectiveTransport, LocalTransport, SeqParallelAttention
    topk = wl.topk[0]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    inp = make_inputs(wl, seed=0)
    nl = wl.N // world
    shard = {n: inp[n][:, rank * nl:(rank + 1) * nl].contiguous().to(dev) for n in ("q", "k", "v")}
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    sp = SeqParallelAttention(rank, world, wl.B, wl.N, wl.H, wl.D, wl.grid, wl.block, topk, gq, gk, wl.rope_split,
                              wl.rope_theta, wl.eps, device=dev)
    transport = LocalTransport() if world == 1 else CollectiveTransport()
    out = torch.empty_like(shard["q"])

    def step(ev=None):
        marks = []
        def mark():
            if ev is not None:
                ev[len(marks)].record(stream)
            marks.append(0)
        mark()
        sp.stage_pack(shard["q"], shard["k"], shard["v"])
        mark()
        sp.exchange_qkv(transport)
        mark()
        sp.stage_compute()
        mark()
        sp.exchange_o(transport)
        mark()
        sp.stage_unpack(out)
        mark()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        barrier(world)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for s_ in range(args.steps):
            step(evs[s_])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    if sol.sol_check_device_status() != sol.SOL_OK:
        raise RuntimeError("device-side error in the timed region")
    ms = max_over_ranks(start.elapsed_time(stop) / args.steps, world)
    names = ("pack_qkv", "exchange_qkv", "compute", "exchange_o", "unpack_o")
    st = {n: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i, n in enumerate(names)}
    flops = wl.selected_flops(topk)
    peaks = load_peaks()
    p = sp.plan
    rows_in = wl.B * nl * wl.H                       # this rank's token-shard rows per tensor
    pack_b = 3 * rows_in * (wl.D * 2 + wl.D + 4)     # read bf16, write codes + scale
    unpack_qkv_b = 3 * p.G * p.rows * (wl.D + 4 + wl.D * 2)
    clocks = sampler.summary()
    if rank != 0:
        return
    line = {
        "metric": "sparse-attn effective TFLOP/s (selected FLOPs)", "value": flops / (ms * 1e-3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "config_id": wl.config_id, "B": wl.B, "N": wl.N, "H": wl.H, "D": wl.D,
                   "grid": list(wl.grid), "block": wl.block, "topk": topk,
                   "parallelism": f"sequence-parallel x{world}: INT8 Q/K/V and FP8 O all-to-all "
                                  f"({'local copy' if world == 1 else 'NCCL'})"},
        "stages_ms": st,
        "pack_qkv": {"GB/s": pack_b / st["pack_qkv"] / 1e6, "frac_hbm": pack_b / st["pack_qkv"] / 1e6 / peaks["hbm_gbs"]},
        "wire_bytes_per_rank": p.wire_bytes(), "bf16_wire_bytes_per_rank": p.bf16_wire_bytes(),
        "unpack_qkv_bytes": unpack_qkv_b,
        "gpu_launches": 11 * args.steps,       # 3 packs, 3 unpacks, the 3-kernel chain, O pack + unpack
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=4, help="workload id (1-4 bf16)")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=0)
    ap.add_argument("--cpu-units", type=int, default=640, help="oracle attention units for cpu_baseline (~12 s)")
    ap.add_argument("--ref-units", type=int, default=24)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="profiling runs: skip the end-to-end runs")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 attention comparison")
    ap.add_argument("--no-per-config", action="store_true", help="skip timing the other bf16 workloads")
    ap.add_argument("--per-config-steps", type=int, default=10)
    ap.add_argument("--backward", action="store_true", help="also time the backward pass (one call)")
    ap.add_argument("--variants", action="store_true",
                    help="also time the selection variants, count-limited attention and 3-D tile blocks")
    ap.add_argument("--chain", choices=("fused", "split"), default="fused",
                    help="fused: prologue emits the block means (3 launches per step); split: the selection "
                         "pools q and k itself (4 launches)")
    ap.add_argument("--parallel", choices=("clips", "seqpar"), default="clips",
                    help="clips: an independent clip per rank (default); seqpar: one clip over all ranks with "
                         "a quantised all-to-all around the path")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.config]
    if wl.dtype != "bf16":
        ap.error("the benchmark runs the bf16 workloads 1-4")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, wl, world, rank)
        elif args.parallel == "seqpar":
            run_seqpar(args, wl, world, rank, local)
        else:
            run_ours(args, wl, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
