"""Benchmark of the fused DPO head step on B200 through libdpo's C ABI.

One step = policy dpo_seq_logprobs(want_grad=1) + reference dpo_seq_logprobs
+ dpo_loss + dpo_backward, on the Llama-3.1-8B head shape (8 rows = 4
chosen/rejected pairs, L = 2048, d = 4096, V = 128,256, bf16), synthetic seeded
inputs. Under torchrun each rank runs its own pairs (data parallel, weak
scaling) with the same weights: the loss call gets the whole batch's pair count
(each rank's loss and coefficients are its share), and the backward forms dW by
blocks of vocabulary rows, each block's NCCL all-reduce running while the next
block is formed, then dH; one small all-reduce sums the loss shares.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 and no torchrun environment, the script starts its own N ranks
(torch.distributed.run on this node) and runs inside them. Rank 0 prints one JSON
line. The value is scored completion tokens per second over all ranks (max time
over ranks, CUDA events, inputs resident in HBM); the K-step loop is timed --reps
times and the median repetition is reported, with the spread and each repetition's
SM clock.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from preference_alignment_b200 import workloads as WL  # noqa: E402

METRIC = "DPO fwd+bwd tokens/s on 1 B200; % of bf16 dense tensor-core peak"
UNIT = "tokens/s"
WORKLOAD = "llama8b"
CONFIG_TEXT = ("Llama-3.1-8B head shape: 4 pairs -> 8 rows, seq 2048, prompt U{256..1024}, "
               "completion to >=95% fill, d=4096, V=128256, bf16; policy fwd+bwd, reference fwd")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dh_parts(Nc, d, V, pairs=74):
    """K parts of the library's dH = dz.W for Nc positions (its plan, restated for the
    launch count): 1, or the vocabulary split into parts of one launch when they fill the
    rounds of 74 CTA pairs better by the plan's estimate (0 when there is nothing to do)."""
    kb = -(-V // 64)
    tiles = -(-Nc // 256) * -(-d // 256)
    if tiles == 0:
        return 0

    def est(units, k):
        return -(-units // pairs) * max(k, 8)

    best, parts = est(tiles, kb), 1
    for q in range(2, 17):
        kbp = -(-kb // q)
        if kbp > (1 << 20) // 64:
            continue
        if kbp < 8:
            break
        n = -(-kb // kbp)
        e = est(tiles * n, kbp) * (1.0 + 0.02 * (n - 1))
        if e < best * 0.97:
            best, parts = e, n
    return parts


def dh_launches(Nc, d, V):
    """Kernel launches of the library's dH: one split launch plus its reduce kernel, or one
    launch over the vocabulary (in chunks of 2^20 columns beyond that)."""
    parts = dh_parts(Nc, d, V)
    if parts == 0:
        return 0
    return 2 if parts > 1 else -(-V // (1 << 20))


# ------------------------------------------------------------------ helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return PEAKS_FALLBACK, "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(argv, n):
    """Re-run this script as n local ranks under torch.distributed.run (one process per
    GPU); returns the launcher's exit status. NCCL's init log stays on (INFO, to stderr,
    so stdout keeps only rank 0's JSON line) and shows the communicator's ranks, unless
    NCCL_DEBUG is already set."""
    env = dict(os.environ)
    if "NCCL_DEBUG" not in env:
        env["NCCL_DEBUG"] = "INFO"
        env.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
        env.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}",
           os.path.abspath(__file__), *argv]
    return subprocess.run(cmd, env=env).returncode


def rank_workload(name, rank, weights=True):
    """The named workload with this rank's own batch (same weights on every rank).

    With weights=False a rank > 0 draws only its batch (W and W_ref are None) and
    receives the weights from rank 0."""
    if rank > 0 and not weights:
        idx, R, L, d, V, dtype, layout, ref_std, rule, has_ref = WL.CONFIGS[name]
        w = WL.Workload(name, R, L, d, V, dtype, layout, 0.1, None, None, None, None, None, None,
                        WL.SEED_BASE + idx)
    else:
        w = WL.make_config(name)
    if rank == 0:
        return w
    idx, R, L, d, V, dtype, layout, ref_std, rule, _ = WL.CONFIGS[name]
    rng = np.random.Generator(np.random.PCG64([w.seed, rank]))
    P, C = rule(rng, R, L)
    w.prompt_len = P.astype(np.int32)
    w.completion_len = C.astype(np.int32)
    w.tokens = rng.integers(0, V, size=(R, L), dtype=np.int64).astype(np.int32)
    w.H = WL.encode(rng.standard_normal(size=(R, L, d), dtype=np.float32), w.dtype)
    return w


def keep_pairs(w, pairs):
    """The workload cut to its first `pairs` pairs (both rows of each), same weights."""
    B = w.R // 2
    if w.layout == "halves":
        rows = np.r_[0:pairs, B:B + pairs]
    else:
        rows = np.arange(2 * pairs)
    w.R = 2 * pairs
    for k in ("prompt_len", "completion_len", "tokens", "H"):
        setattr(w, k, np.ascontiguousarray(getattr(w, k)[rows]))
    return w


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"dpo_bench_clocks_{os.getpid()}_{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v.lower() == "active"})
        sm = [r[0] for r in rows]
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


def cublas_sustained(torch, dev, stream, seconds=1.5, n=8192):
    """bf16 torch.matmul (cuBLAS) back to back for `seconds`: TFLOP/s and the SM clock seen.

    Context only (same GPU, same moment); the roofline uses MEASURED_PEAKS.json."""
    a = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    b = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    c = torch.empty(n, n, device=dev, dtype=torch.bfloat16)
    for _ in range(3):
        torch.matmul(a, b, out=c)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index)
    sampler.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    iters, t0 = 0, time.perf_counter()
    e0.record(stream)
    while time.perf_counter() - t0 < seconds:
        for _ in range(10):
            torch.matmul(a, b, out=c)
        iters += 10
        torch.cuda.synchronize(dev)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = sampler.stop()
    ms = e0.elapsed_time(e1)
    del a, b, c
    return {"tflops": 2.0 * n ** 3 * iters / (ms / 1e3) / 1e12, "n": n, "seconds": ms / 1e3,
            "sm_mhz": clk["sm_mhz"] if clk else None,
            "note": "torch.matmul bf16, same GPU, after the timed regions; context only"}


PROFILED_SOURCES = ["preference_alignment_b200/csrc/" + f for f in
                    ("tc_gemm.cuh", "gemm_launch.cuh", "ptx_sm100.cuh", "tile_config.h", "fwd.cu")]


def kernel_source_hash():
    """Hash of the profiled kernel sources' code: comments, blank lines and trailing
    spaces are dropped first, so only a change of code makes the counters stale."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in PROFILED_SOURCES:
        with open(os.path.join(ROOT, f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(code.encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per launch of the forward GEMM from the committed ncu summary, if the
    kernel sources are unchanged since the counters were taken (else None)."""
    path = os.path.join(ROOT, "profiles", f"fwd_lse_gemm_{workload}_dram.md")
    try:
        vals = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    vals[k.strip()] = v.strip().strip("`")
        if vals.get("source-hash") != kernel_source_hash():
            return None
        return float(vals["dram-bytes-per-launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ oracle sample (host cores)
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


class OracleSample:
    """The CPU fp64 oracle on a bounded sample of the workload: one pair (a chosen
    and a rejected row) with its completions cut to `per_row` tokens each, full
    d and V: policy forward, reference forward, loss and backward to dH and dW,
    the same work per token as the GPU step."""

    def __init__(self, w, per_row):
        from oracle import dpo_oracle as O
        self.O = O
        self.w = w
        B = w.R // 2
        rows = [0, B] if w.layout == "halves" else [0, 1]
        self.H = WL.widen(w.H[rows], w.dtype)
        self.tokens = w.tokens[rows]
        self.P = w.prompt_len[rows].copy()
        self.C = np.minimum(w.completion_len[rows], per_row).astype(np.int32)
        self.W = WL.widen(w.W, w.dtype)
        self.Wr = WL.widen(w.W_ref, w.dtype) if w.W_ref is not None else None
        self.n_tokens = int(self.C.sum())

    def step(self):
        O = self.O
        pol = O.seq_logprobs(self.H, self.W, self.tokens, self.P, self.C)["seq_logp"]
        if self.Wr is None:
            return
        ref = O.seq_logprobs(self.H, self.Wr, self.tokens, self.P, self.C)["seq_logp"]
        lo = O.dpo_loss(pol, ref, self.w.beta, "halves")
        O.backward(self.H, self.W, self.tokens, self.P, self.C, lo["row_coef"])


def run_reference(args):
    """The oracle as the reference arm: K timed steps of a bounded sample on host cores."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = WL.make_config(args.workload)
    s = OracleSample(w, per_row=args.cpu_tokens_per_row)
    for _ in range(args.warmup):
        s.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.step()
    dt = time.perf_counter() - t0
    value = s.n_tokens * args.steps / dt
    cores = blas_threads()
    sample = (f"oracle fp64 (numpy/OpenBLAS) on one pair of the {args.workload} workload, "
              f"completions cut to {args.cpu_tokens_per_row} tokens per row ({s.n_tokens} tokens/step), "
              f"full d and V; policy fwd + reference fwd + loss + backward")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": max(ws, args.gpus),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.workload, "text": CONFIG_TEXT},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(w, per_row):
    s = OracleSample(w, per_row=per_row)
    s.step()                                   # warm caches / page in the widened weights
    t0 = time.perf_counter()
    n = 0
    while True:
        s.step()
        n += 1
        if time.perf_counter() - t0 > 8.0 or n >= 3:
            break
    dt = time.perf_counter() - t0
    return {"value": s.n_tokens * n / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"oracle fp64 on one pair of the {w.name} workload with completions cut to "
                       f"{per_row} tokens per row ({s.n_tokens} tokens), full d={w.d} and V={w.V}; "
                       f"policy fwd + reference fwd + loss + backward; {n} timed repetitions")}


# ------------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from preference_alignment_b200 import dp as DP
    from preference_alignment_b200 import libdpo

    ws_n, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # the data-parallel step (exact shares, dW exchanged by blocks while the next block is
    # formed) runs whenever there are several ranks; --dp-path runs it on one rank too (a
    # one-rank NCCL group), which measures what its structure costs the GPU's compute
    exch = ws_n > 1 or args.dp_path
    if exch:
        import datetime
        # NCCL's own messages (its version line, any debug log) go to stderr, so stdout
        # holds only rank 0's JSON line
        os.environ.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")
        if ws_n == 1:
            store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
            dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                                    timeout=datetime.timedelta(seconds=120), device_id=dev)
        else:
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=dev)
    libdpo.load()
    libdpo.set_gemm_variant(args.gemm_variant)

    w = rank_workload(args.workload, rank, weights=(ws_n == 1 or rank == 0))
    if args.pairs and args.pairs < w.R // 2:
        w = keep_pairs(w, args.pairs)
    B = w.R // 2

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    # offline reference scoring is forward only; a profiler's forward-only run of another
    # workload allocates only what the policy forward needs
    fwd_only = not WL.CONFIGS[args.workload][9] or (args.profile_step > 0 and args.forward_only)
    H = dev_bf16(w.H)
    if ws_n > 1:
        # rank 0 drew the weights; the other ranks receive them (same model on every rank)
        W = dev_bf16(w.W) if rank == 0 else torch.empty(w.V, w.d, dtype=torch.bfloat16, device=dev)
        dist.broadcast(W, 0)
        Wr = None
        if not fwd_only:
            Wr = dev_bf16(w.W_ref) if rank == 0 else torch.empty_like(W)
            dist.broadcast(Wr, 0)
    else:
        W = dev_bf16(w.W)
        Wr = dev_bf16(w.W_ref) if not fwd_only else None
    tokens = torch.from_numpy(w.tokens).to(dev)
    bp = libdpo.BatchArgs(H, W, tokens, w.prompt_len, w.completion_len, dtype="bf16")
    br = libdpo.BatchArgs(H, Wr, tokens, w.prompt_len, w.completion_len, dtype="bf16") if not fwd_only else None
    fwd_b, bwd_b, _ = libdpo.workspace_size(bp)
    ws = torch.empty(fwd_b if fwd_only else max(fwd_b, bwd_b), dtype=torch.uint8, device=dev)
    Nc = w.n_scored
    pol = torch.empty(w.R, device=dev)
    ref = torch.empty(w.R, device=dev)
    lse = torch.empty(Nc, device=dev)
    dH = torch.empty(w.R, w.L, w.d, device=dev) if not fwd_only else None
    scatter = None
    if exch and args.dw_exchange == "scatter" and not fwd_only:
        # dW reduce-scattered inside the dW GEMM: each rank ends with its block of rows
        scatter = DP.FusedReduceScatter(w.V, w.d, device=dev)
        dW = torch.empty(len(scatter.rows), w.d, device=dev)
    else:
        dW = torch.empty(w.V, w.d, device=dev) if not fwd_only else None
    outs = {k: torch.empty(n, device=dev) for k, n in
            [("loss", 1), ("accuracy", 1), ("margins", B), ("cr", B), ("rr", B), ("w", B),
             ("coef", 2 * B)]}
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    # data parallel: the loss is the mean over the whole batch of every rank. Each rank's
    # loss call gets the whole batch's pair count, so its loss, accuracy and row
    # coefficients are its share; one all-reduce sums the shares, the bucketed backward
    # sums dW.
    pairs_total = DP.global_counts(B, 0, device=dev)[0] if exch else 0
    shares = torch.empty(2, device=dev)
    outs["loss"], outs["accuracy"] = shares[0:1], shares[1:2]

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]

    def step(timed=None):
        step_with(bp, br, timed)

    def step_with(bp, br, timed=None, ref_sums=None):
        """One step; with ref_sums (stored reference sums) the reference forward is
        skipped, as in training on offline-scored reference log-probs."""
        if fwd_only:
            if timed is not None:
                ev[0].record(stream)
            libdpo.seq_logprobs(bp, False, pol, None, None, ws, stream=sp)
            if timed is not None:
                ev[1].record(stream)
                torch.cuda.synchronize(dev)
                timed.append([ev[0].elapsed_time(ev[1])] * 2 + [0.0, 0.0])
            return
        if timed is not None:
            ev[0].record(stream)
        libdpo.seq_logprobs(bp, True, pol, None, lse, ws, stream=sp)
        if timed is not None:
            ev[1].record(stream)
        if ref_sums is None:
            libdpo.seq_logprobs(br, False, ref, None, None, ws, stream=sp)
        if timed is not None:
            ev[2].record(stream)
        libdpo.loss_ex(B, w.layout, pol, ref if ref_sums is None else ref_sums, w.beta, 1.0,
                       outs["loss"], outs["accuracy"],
                       outs["margins"], outs["cr"], outs["rr"], outs["w"], outs["coef"],
                       pairs_total=pairs_total, stream=sp)
        if timed is not None:
            ev[3].record(stream)
        if scatter is not None:
            scatter.backward(bp, lse, outs["coef"], dH, dW, ws,
                             max_sms=max(2, sms - args.comm_sms))
            DP.allreduce_shares(shares)
        elif exch:
            works = DP.backward_exchange(bp, lse, outs["coef"], dH, dW, ws,
                                         n_buckets=args.dw_buckets,
                                         max_sms=max(2, sms - args.comm_sms))
            DP.finish(works)
            DP.allreduce_shares(shares)
        else:
            libdpo.backward(bp, lse, outs["coef"], dH, dW, False, ws, stream=sp)
        if timed is not None:
            ev[4].record(stream)
            torch.cuda.synchronize(dev)
            timed.append([ev[i].elapsed_time(ev[i + 1]) for i in range(4)])

    # launches of our kernels per step: upload + prep + GEMM + combine + rowsum per forward,
    # one loss kernel; the backward (one token chunk: the workspace holds all Nc rows of
    # dz) runs upload + prep + the dz GEMM + the dH launches (dh_launches) + the dW GEMM
    uploads = math.ceil(w.R / 1024)
    fwd_launches = uploads + 4
    n_dh = dh_launches(Nc, w.d, w.V)
    if scatter is not None:   # dz, the scatter dW GEMM, dH, the owner's sum of its slots
        bwd_launches = uploads + 2 + 1 + n_dh + 1
    elif exch:     # dz, then dW by blocks of vocabulary rows, then dH
        bwd_launches = uploads + 2 + len(DP.vocab_buckets(w.V, args.dw_buckets)) + n_dh
    else:
        bwd_launches = uploads + 3 + n_dh
    launches_per_step = (fwd_launches if fwd_only else 2 * fwd_launches + 1 + bwd_launches)

    if args.profile_step:
        # a profiler's run: the given number of plain steps, nothing timed or printed (a
        # forward-only run also makes one dpo_logits_mean call: it needs only H, W and the
        # forward workspace)
        for _ in range(args.profile_step):
            step()
        if args.forward_only:
            libdpo.logits_mean(bp, w.layout, torch.empty(2, device=dev), ws, stream=sp)
        st = libdpo.check(sp)
        if exch:
            if scatter is not None:
                dist.barrier()
                scatter.close()
            dist.destroy_process_group()
        return 0 if st == libdpo.OK else 1

    for _ in range(args.warmup):
        step()
    st = libdpo.check(sp)
    if st != libdpo.OK:
        raise RuntimeError(f"device status after warm-up: {libdpo.status_string(st)}")

    # per-call breakdown (separate short pass with a sync after each step)
    breakdown = []
    for _ in range(min(5, args.steps)):
        step(timed=breakdown)
    bd = np.median(np.array(breakdown), axis=0)

    # the K-step loop, timed args.reps times: barrier + synchronize on both sides of each
    # repetition, CUDA events on the launching stream, clocks sampled during each one
    rep_ms, rep_clk = [], []
    for _ in range(args.reps):
        clocks = ClockSampler(local)
        if ws_n > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        clocks.start()
        time.sleep(0.3)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for _ in range(args.steps):
            step()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if ws_n > 1:
            dist.barrier()
        rep_clk.append(clocks.stop())
        rep_ms.append(t_start.elapsed_time(t_end))
    st = libdpo.check(sp)
    if st != libdpo.OK:
        raise RuntimeError(f"device status after timing: {libdpo.status_string(st)}")

    # ------------------------------------------------------------ offline-scored reference
    # The same step with the reference sums read from storage instead of a reference
    # forward (the reference scored once, offline): policy forward, loss, backward.
    offline_ms = None
    if not fwd_only:
        ref_stored = ref.clone()
        for _ in range(2):
            step_with(bp, br, ref_sums=ref_stored)
        if ws_n > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        o0 = torch.cuda.Event(enable_timing=True)
        o1 = torch.cuda.Event(enable_timing=True)
        o0.record(stream)
        for _ in range(args.steps):
            step_with(bp, br, ref_sums=ref_stored)
        o1.record(stream)
        torch.cuda.synchronize(dev)
        if ws_n > 1:
            dist.barrier()
        offline_ms = o0.elapsed_time(o1)

    # ------------------------------------------------------------ end to end (host buffers)
    # Every step uploads its inputs (H, tokens) from pinned host memory and reads its
    # results (loss and metrics) back. As a training loop would, the upload of step
    # i + 1 runs on a copy stream into the other of two input buffers while step i
    # computes (the step waits for its own upload with an event), and the host reads
    # step i's results once step i + 1 is queued behind it, so the GPU never idles
    # while the host waits for a result.
    H_host = torch.from_numpy(np.ascontiguousarray(w.H).view(np.int16)).view(torch.bfloat16).pin_memory()
    tok_host = torch.from_numpy(w.tokens).pin_memory()
    res_host = torch.empty(2, max(2 + 3 * B, w.R), dtype=torch.float32).pin_memory()
    res_ready = [torch.cuda.Event() for _ in range(2)]
    host_read = []
    e2e_steps = max(3, min(args.steps, 20))
    copy_stream = torch.cuda.Stream(dev)
    H_buf = [H, torch.empty_like(H)]
    tok_buf = [tokens, torch.empty_like(tokens)]
    batches = []
    for i in range(2):
        if fwd_only:
            batches.append((libdpo.BatchArgs(H_buf[i], W, tok_buf[i], w.prompt_len, w.completion_len,
                                             dtype="bf16"), None))
        else:
            batches.append((libdpo.BatchArgs(H_buf[i], W, tok_buf[i], w.prompt_len, w.completion_len,
                                             dtype="bf16"),
                            libdpo.BatchArgs(H_buf[i], Wr, tok_buf[i], w.prompt_len, w.completion_len,
                                             dtype="bf16")))
    uploaded = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def upload(i):
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(consumed[i % 2])          # buffer free again
            H_buf[i % 2].copy_(H_host, non_blocking=True)
            tok_buf[i % 2].copy_(tok_host, non_blocking=True)
            uploaded[i % 2].record(copy_stream)

    for i in range(2):
        consumed[i].record(stream)
    e2e_reps = []
    for _ in range(args.reps):
        if ws_n > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        upload(0)
        for i in range(e2e_steps):
            if i + 1 < e2e_steps:
                upload(i + 1)
            stream.wait_event(uploaded[i % 2])
            bp_i, br_i = batches[i % 2]
            step_with(bp_i, br_i)
            consumed[i % 2].record(stream)
            if fwd_only:
                res_dev = pol
            else:
                res_dev = torch.cat([outs["loss"], outs["accuracy"], outs["margins"], outs["cr"],
                                     outs["rr"]])
            res_host[i % 2, :res_dev.numel()].copy_(res_dev, non_blocking=True)
            res_ready[i % 2].record(stream)
            if i > 0:                                        # the host reads step i - 1
                res_ready[(i - 1) % 2].synchronize()
                host_read.append(float(res_host[(i - 1) % 2, 0]))
        res_ready[(e2e_steps - 1) % 2].synchronize()         # and the last step
        host_read.append(float(res_host[(e2e_steps - 1) % 2, 0]))
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_reps.append(e0.elapsed_time(e1))
    h2d = H_host.numel() * 2 + tok_host.numel() * 4
    d2h = (w.R if fwd_only else 2 + 3 * B) * 4

    # ------------------------------------------------------------ logits-mean metrics
    # dpo_logits_mean (not part of the step): two HBM-bound column sums (W, then each
    # side's H rows) and a dot product; algorithmic bytes = W + H read once.
    lm_means = torch.empty(2, device=dev)
    for _ in range(3):
        libdpo.logits_mean(bp, w.layout, lm_means, ws, stream=sp)
    lm_reps = 10
    l0 = torch.cuda.Event(enable_timing=True)
    l1 = torch.cuda.Event(enable_timing=True)
    l0.record(stream)
    for _ in range(lm_reps):
        libdpo.logits_mean(bp, w.layout, lm_means, ws, stream=sp)
    l1.record(stream)
    torch.cuda.synchronize(dev)
    lm_ms = l0.elapsed_time(l1) / lm_reps
    lm_bytes = 2 * (w.V * w.d + w.R * w.L * w.d)

    # ------------------------------------------------------------ same-box cuBLAS reference
    cublas = None
    if not args.no_cublas_reference:
        cublas = cublas_sustained(torch, dev, stream, seconds=1.5)

    # ------------------------------------------------------------ aggregate over ranks
    # each repetition's time is the max over ranks; the median repetition is reported
    t = torch.tensor(rep_ms + e2e_reps + [offline_ms or 0.0, float(Nc)], device=dev,
                     dtype=torch.float64)
    if ws_n > 1:
        tmax = t.clone()
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
        tsum = t.clone()
        dist.all_reduce(tsum, op=dist.ReduceOp.SUM)
        rep_ms = [float(x) for x in tmax[:args.reps]]
        e2e_reps = [float(x) for x in tmax[args.reps:2 * args.reps]]
        if offline_ms is not None:
            offline_ms = float(tmax[-2])
        total_nc = float(tsum[-1])
    else:
        total_nc = float(Nc)
    order = sorted(range(args.reps), key=lambda i: rep_ms[i])
    med = order[(args.reps - 1) // 2]                 # the median repetition (lower middle)
    ms = rep_ms[med]
    clk = dict(rep_clk[med]) if rep_clk[med] else None
    if clk is not None:        # throttle reasons seen in any repetition
        clk["reasons"] = sorted({r for c in rep_clk if c for r in c["reasons"]})
    e2e_ms = sorted(e2e_reps)[(args.reps - 1) // 2]
    rep_mhz = [c["sm_mhz"] if c else None for c in rep_clk]

    peaks, peak_src = load_peaks()
    value = total_nc * args.steps / (ms / 1e3)
    e2e_value = total_nc * e2e_steps / (e2e_ms / 1e3)
    ms_step = ms / args.steps
    gemm_flop = 2.0 * Nc * w.d * w.V                      # one LM-head GEMM over scored tokens
    alg_flop = (1 if fwd_only else 4) * gemm_flop          # policy fwd, ref fwd, dH, dW
    exe_flop = (1 if fwd_only else 5) * gemm_flop          # + backward logit recompute
    sustained = float(peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]))
    hbm_peak = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    # dominant kernel: the forward LSE GEMM (two launches per step), timed by the events
    # around the reference dpo_seq_logprobs call (the call also runs the small prep,
    # combine and row-sum kernels, so the figure is a slight underestimate)
    fwd_ms = float(bd[1])
    fwd_tflops = gemm_flop / (fwd_ms / 1e3) / 1e12
    line = None
    if rank == 0:
        cpu = None
        if ws_n == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(w, per_row=args.cpu_tokens_per_row)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; random-init LM-head weights of the Llama-3.1-8B head shape)",
            "config": {"workload": args.workload, "text": CONFIG_TEXT, "rows_per_gpu": w.R,
                       "gemm_variant_mask": args.gemm_variant,
                       "pairs_per_gpu": B, "seq_len": w.L, "d": w.d, "V": w.V,
                       "scored_tokens_per_gpu": Nc, "global_batch_pairs": B * ws_n,
                       "parallelism": f"dp{ws_n}",
                       "dw_exchange": (None if not exch else
                                       f"reduce-scatter fused into the dW GEMM (CUDA IPC "
                                       f"receive buffers), {args.comm_sms} SMs left free"
                                       if scatter is not None else
                                       f"all-reduce of {args.dw_buckets} blocks of vocabulary "
                                       f"rows, {args.comm_sms} SMs left to NCCL"),
                       "l2": "inputs larger than L2 (W and W_ref are 1.05 GB each; no flush)"},
            "pct_of_peak": {"algorithmic": alg_flop * args.steps / (ms / 1e3) / 1e12 / sustained,
                            "executed": exe_flop * args.steps / (ms / 1e3) / 1e12 / sustained,
                            "peak_tflops": sustained, "peak": f"bf16 sustained, {peak_src}",
                            "flop_per_step_algorithmic": alg_flop,
                            "flop_per_step_executed": exe_flop,
                            # the same throughput against the other denominators in use
                            "other_peaks": {
                                name: {"tflops": pk,
                                       "algorithmic": alg_flop * args.steps / (ms / 1e3) / 1e12 / pk,
                                       "executed": exe_flop * args.steps / (ms / 1e3) / 1e12 / pk}
                                for name, pk in (
                                    (f"bf16 burst, {peak_src}",
                                     float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))),
                                    ("bf16 dense datasheet (nominal, not reachable under the "
                                     "1 kW cap)", 2250.0))}},
            "batch_tokens_per_s": w.R * w.L * ws_n * args.steps / (ms / 1e3),
            "breakdown_ms": {"policy_fwd": float(bd[0]), "ref_fwd": float(bd[1]),
                             "loss": float(bd[2]), "backward": float(bd[3])},
            "roofline": {"kernel": "k_tc_gemm_pair<EpiLSE> (forward LM-head GEMM + online LSE)",
                         "bound": "tensor", "achieved": fwd_tflops, "peak": sustained,
                         "unit": "TFLOP/s", "frac": fwd_tflops / sustained,
                         "traffic": profiled_traffic(args.workload),
                         "algorithmic_per_launch": f"2*Nc*d*V = {gemm_flop:.4g} FLOP",
                         "peak_kind": f"bf16_tflops_sustained ({peak_src})"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "repeats": {
                "n": args.reps, "reported": "median repetition",
                "ms_per_step": [x / args.steps for x in rep_ms],
                "sm_mhz": rep_mhz,
                "spread_pct": 100.0 * (max(rep_ms) - min(rep_ms)) / ms,
                "ms_x_ghz_per_step": [x / args.steps * m / 1e3 if m else None
                                      for x, m in zip(rep_ms, rep_mhz)],
                "e2e_ms_per_step": [x / e2e_steps for x in e2e_reps],
                "reasons": sorted({r for c in rep_clk if c for r in c["reasons"]}),
            },
            "cpu_baseline": cpu,
            "cublas_same_box": cublas,
            "offline_reference_step": None if offline_ms is None else {
                "ms_per_step": offline_ms / args.steps,
                "value": total_nc * args.steps / (offline_ms / 1e3), "unit": UNIT,
                "gemms_per_step": 4,
                "pct_of_peak_executed": 4 * gemm_flop * args.steps / (offline_ms / 1e3) / 1e12
                                        / sustained,
                "note": "policy forward + loss on stored reference sums + backward (reference "
                        "scored offline); one timed loop right after the main repetitions"},
            "logits_mean_metric": {"ms": lm_ms, "bytes": lm_bytes,
                                   "GB/s": lm_bytes / (lm_ms / 1e3) / 1e9,
                                   "frac": lm_bytes / (lm_ms / 1e3) / 1e9 / hbm_peak,
                                   "peak_gbs": hbm_peak, "bound": "hbm",
                                   "note": "dpo_logits_mean, not part of the step; W and H read once"},
            "peak_device_bytes": torch.cuda.max_memory_allocated(dev),
            "logits_fp32_bytes_avoided": 4 * Nc * w.V,
        }
        print(json.dumps(line), flush=True)
    if exch:
        if scatter is not None:
            torch.cuda.synchronize(dev)
            dist.barrier()
            scatter.close()
        if ws_n > 1:
            dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(WL.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cublas-reference", action="store_true")
    ap.add_argument("--gemm-variant", type=int, default=0, choices=range(512),
                    help="mask, per GEMM (forward, dz, dH, dW) bit k: single-CTA kernel, "
                         "bit 4 + k: static tile schedule; bit 8: dH without split-K")
    ap.add_argument("--cpu-tokens-per-row", type=int, default=64,
                    help="oracle sample (CPU baseline and reference arm): completion tokens "
                         "per row of one pair")
    ap.add_argument("--reps", type=int, default=5,
                    help="repetitions of the timed K-step loop (the median is reported)")
    ap.add_argument("--dw-buckets", type=int, default=8,
                    help="data parallel: blocks of dW rows whose all-reduce overlaps the next")
    ap.add_argument("--comm-sms", type=int, default=16,
                    help="data parallel: SMs the backward GEMMs leave free for NCCL")
    ap.add_argument("--dw-exchange", choices=["allreduce", "scatter"], default="allreduce",
                    help="data parallel: NCCL all-reduce of dW blocks overlapped with the "
                         "backward, or the reduce-scatter fused into the dW GEMM")
    ap.add_argument("--dp-path", action="store_true",
                    help="run the data-parallel step (bucketed dW exchange) on a single rank "
                         "too, to measure what its structure costs")
    ap.add_argument("--pairs", type=int, default=0,
                    help="keep only the workload's first P pairs (a smaller case, e.g. for a "
                         "profiler); 0 = all")
    ap.add_argument("--profile-step", type=int, default=0,
                    help="run this many untimed steps and exit (a profiler's command)")
    ap.add_argument("--forward-only", action="store_true",
                    help="with --profile-step: the policy forward alone, then one logits-mean "
                         "call (weights, H and the forward workspace on the device, nothing else)")
    raw = sys.argv[1:] if argv is None else list(argv)
    args = ap.parse_args(raw)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    args.reps = max(1, args.reps)
    ws = int(os.environ.get("WORLD_SIZE", "0"))
    if ws == 0 and args.gpus > 1:
        return launch_ranks(raw, args.gpus)
    if ws > 0 and ws != args.gpus:
        print(f"bench.py: WORLD_SIZE={ws} but --gpus {args.gpus}", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
