"""Benchmark of the gated delta rule forward on B200.

python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

One step = one gdr_chunk_fwd call over the whole workload (cumulative decay, WY
construction, state propagation and output for every chunk of every sequence-
head), inputs resident in HBM.  Workloads (synthetic, seeded; workload/):
  gdn2_t4k   (default) B=8, H=16, T=4096, dk=dv=128, chunk 64, bf16, Gated DeltaNet-2
  gdn_t2k    B=4, H=16, T=2048, Gated DeltaNet (scalar gates)
  gdn2_t16k  B=1, H=16, T=16384;  gdn2_t16k_kda: the tied KDA mode on the same inputs
  gdn2_t4k_bonly / gdn2_t4k_wonly: the b-only / w-only gate-ablation variants of gdn2_t4k
  mixer_t4k  the T=4K shape through gdr_mixer_fwd: raw token-major projections in, the
             RMSNorm-SiLU-gated output out (activations and epilogue fused in the kernel)
  bwd_t4k    the backward (gdr_chunk_bwd) of gdn2_t4k: dq, dk, dv, dg, db, dw and dS0 from dO
             and dS_T (four launches on the tcgen05 tensor cores; the last, for strong-decay
             spans, has none here)
  decode     256 sequences x 16 heads, one token per step, state in place
Metric: token-heads/s (tokens/s per head-layer) = B*H*T / step time (decode:
step-heads/s).  With N ranks every rank runs its own copy of the workload on its
GPU (sequence-heads are independent: weak scaling, no collective on the data
path) and value = all ranks' units / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workload  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


# ---------------------------------------------------------------------------------------
# algorithmic counts (each input read once, each output written once)
def chunk_bytes(wl: workload.Workload, mode: str) -> float:
    e = 2 if wl.dtype == "bf16" else 4
    dk, dv = wl.dk, wl.dv
    per_tok = (2 * dk + dv) * e + dv * e               # q, k, v in; o out
    if mode == "gdn2":
        per_tok += dk * 4 + dk * e + dv * e             # g [dk] fp32, b [dk], w [dv]
    elif mode == "bonly":
        per_tok += dk * 4 + dk * e + e                  # g [dk], b [dk], scalar w
    elif mode == "wonly":
        per_tok += dk * 4 + e + dv * e                  # g [dk], scalar b, w [dv]
    elif mode == "kda":
        per_tok += dk * 4 + e                           # g [dk], beta
    else:
        per_tok += 4 + e                                # g scalar, beta
    per_head_state = (2 if wl.s0_std > 0 else 1) * dk * dv * 4   # S_T write (+ S0 read)
    return wl.units * per_tok + wl.B * wl.H * per_head_state


def chunk_flops(wl: workload.Workload) -> float:
    """Dense products of the chunkwise form per token-head: 6 dk dv + 10 C d
    (A, P, W, U, W S, Q S, P E, K^T E; the triangular inverse is not counted)."""
    d = max(wl.dk, wl.dv)
    return wl.units * (6.0 * wl.dk * wl.dv + 10.0 * wl.chunk * d)


def mixer_bytes(cfg) -> float:
    """Raw projections read once (q, k, v, xb, xw, z bf16; xg fp32), y written once, S0 read
    and S_T written once per head."""
    dk, dv = cfg["dk"], cfg["dv"]
    per_tok = (2 * dk + dv) * 2 + dk * 4 + dk * 2 + dv * 2 + dv * 2 + dv * 2
    per_head = (2 if cfg["s0_std"] > 0 else 1) * dk * dv * 4
    return cfg["B"] * cfg["H"] * (cfg["T"] * per_tok + per_head)


def bwd_bytes(wl: workload.Workload) -> float:
    """Inputs (q, k, v, g, b, w) and dO read once, the gradients written once, S0 and dS_T
    read and dS0 written once per head (GDN-2, bf16 storage, fp32 g, dg and states)."""
    dk, dv = wl.dk, wl.dv
    per_tok = (2 * dk + dv) * 2 + dk * 4 + dk * 2 + dv * 2 + dv * 2    # q k v g b w dO
    per_tok += (2 * dk + dv) * 2 + dk * 4 + dk * 2 + dv * 2            # dq dk dv dg db dw
    return wl.units * per_tok + wl.B * wl.H * 3 * dk * dv * 4


def bwd_flops(wl: workload.Workload) -> float:
    """Tensor-core products of the backward per token-head, 64-token chunks: 22 d^2 + 40 C d
    (checkpoints: the forward's 6 d^2 + 10 C d; state gradient 6 d^2 + 8 C d; per-chunk
    gradients 10 d^2 + 22 C d, i.e. 5 C d^2 + 11 C^2 d multiply-adds per chunk)."""
    C, d = 64, max(wl.dk, wl.dv)
    return wl.units * (22.0 * d * d + 40.0 * C * d)


def decode_bytes(cfg) -> float:
    e = 2 if cfg["dtype"] == "bf16" else 4
    dk, dv = cfg["dk"], cfg["dv"]
    per = 2 * dk * dv * 4 + (2 * dk + dv) * e + dk * 4 + dk * e + dv * e + dv * e
    return cfg["N"] * cfg["H"] * per


def load_peaks():
    try:
        p = json.load(open(PEAKS_FILE))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ---------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        self.first = ""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        if self.proc is not None:
            # the timed region starts only once the sampler is running: wait (up to 3 s) for its
            # first sample, read from the raw pipe so that communicate() later sees the rest
            import select
            fd, buf, deadline = self.proc.stdout.fileno(), b"", time.time() + 3.0
            while b"\n" not in buf and time.time() < deadline:
                ready, _, _ = select.select([fd], [], [], max(0.0, deadline - time.time()))
                if not ready:
                    break
                chunk = os.read(fd, 4096)
                if not chunk:
                    break
                buf += chunk
            self.first = buf.decode(errors="replace")
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in (self.first + out).splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --batch: a smaller batch of the same sequences, for ncu captures of a small case (the
# workload then reports the batch it ran; never the bench's default)
BATCH = None


def rank_workload(name: str, rank: int):
    """Each rank's own share: the named workload's shape with a rank-specific seed."""
    if name == "decode":
        cfg = dict(workload.DECODE)
        cfg["seed"] = cfg["seed"] + 1000 * rank
        return cfg, "gdn2"
    if name == "mixer_t4k":
        cfg = dict(workload.MIXER)
        cfg["seed"] = cfg["seed"] + 1000 * rank
        return cfg, cfg["mode"]
    if name == "bwd_t4k":
        name = "gdn2_t4k"
    base, mode = name, None
    for m in ("kda", "bonly", "wonly"):
        if name.endswith("_" + m):
            base, mode = name[:-len(m) - 1], m
    from dataclasses import replace
    wl = workload.CONFIGS[base]
    if rank:
        wl = replace(wl, seed=wl.seed + 1000 * rank)
    if BATCH is not None:
        wl = replace(wl, B=BATCH)
    return wl, mode or wl.mode


# ---------------------------------------------------------------------------------------
def cpu_oracle_sample(name, target_cpu_s=15.0):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload."""
    import oracle
    cores = oracle.default_threads()
    if name == "decode":
        cfg = workload.DECODE
        pool = workload.make_decode_pool(cfg, N=16, pool=4)
        S = pool["S0"]
        n_heads = 16 * cfg["H"]
        steps = 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < target_cpu_s / cores and steps < 1000:
            p = steps % 4
            _, S = oracle.decode(pool["q"][p], pool["k"][p], pool["v"][p], pool["g"][p],
                                 pool["b"][p], pool["w"][p], S=S, mode="gdn2", nthreads=cores)
            steps += 1
        dt = time.perf_counter() - t0
        return dict(value=steps * n_heads / dt, unit="step-heads/s", cores=cores, kind="oracle",
                    sample=f"{steps} decode steps of 16 sequences x {cfg['H']} heads (of 256 x {cfg['H']})")
    if name == "mixer_t4k":
        from oracle import mixer
        c = workload.MIXER
        d = workload.make_mixer_inputs(1, 1, c["T"], c["dk"], c["dv"], mode=c["mode"], layout=c["layout"],
                                       seed=c["seed"], xg_shift=c["xg_shift"], s0_std=c["s0_std"])
        t0 = time.perf_counter()
        mixer.mixer_fwd(d["q"], d["k"], d["v"], d["xg"], d["xb"], d["xw"], d["z"], d["weight"], d["S0"],
                        mode=c["mode"], token_major=True)
        t_head = time.perf_counter() - t0
        # a batch of sampled sequence-heads (the same draw repeated), so that the recurrence
        # oracle's threads have one head each
        n = max(cores, int(round(target_cpu_s / max(t_head, 1e-3) / cores)) * cores)
        n = min(n, c["B"] * c["H"])
        rep = lambda x: None if x is None else x.expand(n, *x.shape[1:]).contiguous()
        t0 = time.perf_counter()
        mixer.mixer_fwd(rep(d["q"]), rep(d["k"]), rep(d["v"]), rep(d["xg"]), rep(d["xb"]), rep(d["xw"]),
                        rep(d["z"]), d["weight"], rep(d["S0"]), mode=c["mode"], token_major=True)
        dt = time.perf_counter() - t0
        return dict(value=n * c["T"] / dt, unit="token-heads/s", cores=min(cores, n), kind="oracle",
                    sample=f"{n} sequence-heads x T={c['T']} of mixer_t4k, one batch")
    if name == "bwd_t4k":
        wl, mode = rank_workload(name, 0)
        small = workload.Workload("sample", B=1, H=1, T=wl.T, dk=wl.dk, dv=wl.dv, chunk=wl.chunk,
                                  dtype=wl.dtype, mode=wl.mode, seed=wl.seed, g_scale=wl.g_scale,
                                  s0_std=wl.s0_std)
        d = workload.make_inputs(small, mode=mode)
        gen = torch.Generator().manual_seed(99)
        dO = torch.randn(1, 1, wl.T, wl.dv, generator=gen).to(torch.bfloat16)
        dST = torch.randn(1, 1, wl.dk, wl.dv, generator=gen) * 0.1
        t0 = time.perf_counter()
        oracle.bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], dO, dST, mode=mode, nthreads=1)
        t_head = time.perf_counter() - t0
        n_heads = max(cores, int(round(target_cpu_s / max(t_head, 1e-3) / cores)) * cores)
        n_heads = min(n_heads, wl.B * wl.H)
        rep = lambda x: None if x is None else x.expand(n_heads, *x.shape[1:]).contiguous()
        dd = {k: rep(d[k]) for k in ("q", "k", "v", "g", "b", "w", "S0")}
        t0 = time.perf_counter()
        oracle.bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], rep(dO), rep(dST), mode=mode,
                   nthreads=cores)
        dt = time.perf_counter() - t0
        return dict(value=n_heads * wl.T / dt, unit="token-heads/s", cores=min(cores, n_heads), kind="oracle",
                    sample=f"{n_heads} sequence-heads x T={wl.T} of bwd_t4k (adjoint oracle)")
    wl, mode = rank_workload(name, 0)
    T = wl.T
    small = workload.Workload("sample", B=1, H=1, T=T, dk=wl.dk, dv=wl.dv, chunk=wl.chunk,
                              dtype=wl.dtype, mode=wl.mode, seed=wl.seed, g_scale=wl.g_scale,
                              s0_std=wl.s0_std)
    d = workload.make_inputs(small, mode=mode)
    t0 = time.perf_counter()
    oracle.fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode, nthreads=1)
    t_head = time.perf_counter() - t0
    n_heads = max(cores, int(round(target_cpu_s / max(t_head, 1e-3) / cores)) * cores)
    n_heads = min(n_heads, wl.B * wl.H)
    rep = lambda x: None if x is None else x.expand(n_heads, *x.shape[1:]).contiguous()
    dd = {k: rep(d[k]) for k in ("q", "k", "v", "g", "b", "w", "S0")}
    t0 = time.perf_counter()
    oracle.fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["S0"], mode=mode,
               nthreads=cores)
    dt = time.perf_counter() - t0
    return dict(value=n_heads * T / dt, unit="token-heads/s", cores=min(cores, n_heads),
                kind="oracle", sample=f"{n_heads} sequence-heads x T={T} of {name}")


# ---------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    name = args.workload
    steps_cpu = []
    for _ in range(args.warmup):
        cpu_oracle_sample(name, target_cpu_s=2.0)
    for _ in range(args.steps):
        steps_cpu.append(cpu_oracle_sample(name, target_cpu_s=args.ref_cpu_s))
    v = statistics.median(s["value"] for s in steps_cpu)
    unit = steps_cpu[0]["unit"]
    line = {"impl": "reference", "metric": metric_name(name), "value": v, "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "dtype": "f64", "data": "synthetic",
            "config": config_of(name, world),
            "cpu_baseline": {"value": v, "unit": unit, "cores": steps_cpu[0]["cores"],
                             "kind": "oracle", "sample": steps_cpu[0]["sample"]},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "vs_baseline": None}
    print(json.dumps(line), flush=True)


def metric_name(name):
    if name == "decode":
        return "decode step-heads/s (256 seqs x 16 heads, dk=dv=128); % HBM roofline"
    if name == "mixer_t4k":
        return "token-mixer fwd tokens/s per head·layer at T=4K (fused prologue/epilogue); % HBM roofline"
    if name == "bwd_t4k":
        return "chunked bwd tokens/s per head·layer at T=4K (dq, dk, dv, dg, db, dw, dS0); % HBM roofline"
    return "chunked fwd tokens/s per head·layer at T=4K; % tensor-pipe / HBM roofline"


def config_of(name, world):
    if name == "decode":
        c = workload.DECODE
        return {"workload": "gdn2_decode", "N": c["N"], "H": c["H"], "dk": c["dk"], "dv": c["dv"],
                "mode": "gdn2", "state": "fp32 in place", "inputs": "bf16",
                "l2": "state 537 MB per step > L2", "parallelism": f"replicas{world}"}
    if name == "mixer_t4k":
        c = workload.MIXER
        return {"workload": name, "B": c["B"], "H": c["H"], "T": c["T"], "dk": c["dk"], "dv": c["dv"],
                "chunk": c["chunk"], "mode": c["mode"], "layout": "[B,T,H,D]", "inputs": "bf16 raw projections",
                "state": "fp32", "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas{world}"}
    if name == "bwd_t4k":
        wl, mode = rank_workload(name, 0)
        return {"workload": name, "B": wl.B, "H": wl.H, "T": wl.T, "dk": wl.dk, "dv": wl.dv, "chunk": 64,
                "mode": mode, "inputs": wl.dtype, "state": "fp32", "grad": "dO bf16 N(0,1), dS_T N(0,0.1)",
                "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas{world}"}
    wl, mode = rank_workload(name, 0)
    return {"workload": name, "B": wl.B, "H": wl.H, "T": wl.T, "dk": wl.dk, "dv": wl.dv,
            "chunk": wl.chunk, "mode": mode, "inputs": wl.dtype, "state": "fp32",
            "l2": "inputs larger than L2 (no flush)" if chunk_bytes(wl, mode) > 126e6
            else "L2 flushed between steps", "parallelism": f"replicas{world}"}


def setup_workload(name, rank, dev, decode_steps=None):
    """Inputs resident on `dev` and the callables of one bench step of workload `name`.
    Returns a dict: step (one whole step, L2 flush included), fwd (the timed launches),
    flush (a buffer written between timed launches, or None), units, unit,
    bytes_per_launch, launches_per_step, kernel (name of the timed kernels), flops (tensor
    products per step, or None), nseg, and the host-side inputs for the end-to-end leg."""
    import linear_attention_recurrence_wy_b200 as gdr
    wl, mode = rank_workload(name, rank)
    r = dict(name=name, wl=wl, mode=mode, flush=None, flops=None, nseg=1, unit="token-heads/s")
    if name == "mixer_t4k":
        c = wl
        inp = workload.make_mixer_inputs(c["B"], c["H"], c["T"], c["dk"], c["dv"], mode=c["mode"],
                                         layout=c["layout"], seed=c["seed"], xg_shift=c["xg_shift"],
                                         s0_std=c["s0_std"])
        d = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
        y = torch.empty(c["B"], c["T"], c["H"], c["dv"], dtype=torch.bfloat16, device=dev)
        ST = torch.empty(c["B"], c["H"], c["dk"], c["dv"], dtype=torch.float32, device=dev)

        def fwd():
            gdr.mixer_fwd(d["q"], d["k"], d["v"], d["xg"], d["xb"], d["xw"], d["z"], d["weight"], d["S0"],
                          mode=c["mode"], layout=c["layout"], y=y, S_T=ST)
        r.update(fwd=fwd, step=fwd, units=c["B"] * c["H"] * c["T"], bytes_per_launch=mixer_bytes(c),
                 launches_per_step=1, inp=inp, out=(y, ST),
                 kernel="gdr chunk_tc_kernel<mixer> (tcgen05, fused prologue/epilogue)")
    elif name == "bwd_t4k":
        inp = workload.make_inputs(wl, mode=mode)
        d = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
        gen = torch.Generator().manual_seed(99 + rank)
        dO = torch.randn(wl.B, wl.H, wl.T, wl.dv, generator=gen).to(torch.bfloat16).to(dev)
        dST = (torch.randn(wl.B, wl.H, wl.dk, wl.dv, generator=gen) * 0.1).to(dev)
        ws = torch.empty(gdr.gdr_chunk_bwd_workspace(wl.B, wl.H, wl.T, wl.dk, wl.dv), dtype=torch.uint8,
                         device=dev)
        grads = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]), dv=torch.empty_like(d["v"]),
                     dg=torch.empty_like(d["g"]), db=torch.empty_like(d["b"]), dw=torch.empty_like(d["w"]),
                     dS0=torch.empty_like(d["S0"]))

        def fwd():
            gdr.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], dO, dST, mode=mode,
                          workspace=ws, out=grads)
        # one step = the whole backward (states, state gradient, per-chunk gradients, and the
        # CUDA-core kernel for strong-decay spans, none here), the unit of the roofline
        r.update(fwd=fwd, step=fwd, units=wl.units, bytes_per_launch=bwd_bytes(wl), launches_per_step=4,
                 flops=bwd_flops(wl), inp=inp, dO=dO, dST=dST, ws=ws, grads=grads,
                 kernel="gdr chunk_tc_kernel (checkpoints) + chunk_tc_kernel (state gradient) + "
                        "bwd_tc_kernel + bwd_chunk_kernel (backward, 4 launches, tcgen05)")
    elif name == "decode":
        pool = workload.make_decode_pool(wl)
        d = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in pool.items()}
        S = d["S0"].clone()
        P = wl["pool"]
        n_inner = decode_steps or wl["steps"]

        def step():
            for s_ in range(n_inner):
                p_ = s_ % P
                gdr.decode_step(d["q"][p_], d["k"][p_], d["v"][p_], d["g"][p_], d["b"][p_], d["w"][p_], S,
                                mode="gdn2")
        r.update(fwd=step, step=step, units=wl["N"] * wl["H"] * n_inner, bytes_per_launch=decode_bytes(wl),
                 launches_per_step=n_inner, unit="step-heads/s",
                 kernel="gdr decode_stream_kernel" if wl["dk"] == wl["dv"] == 128 else "gdr decode_kernel")
    else:
        inp = workload.make_inputs(wl, mode=mode)
        d = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
        o = torch.empty(wl.B, wl.H, wl.T, wl.dv, dtype=d["q"].dtype, device=dev)
        ST = torch.empty(wl.B, wl.H, wl.dk, wl.dv, dtype=torch.float32, device=dev)
        flush = None
        if chunk_bytes(wl, mode) <= 126e6:
            flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        dt_code = 1 if wl.dtype == "bf16" else 0
        # the library's planner picks the path: the two-phase forward (few sequence-heads,
        # long sequences), the fused kernel with a sequence split, or the fused kernel alone
        n2 = gdr.gdr_chunk_fwd_two_phase_segments(wl.B, wl.H, wl.T, wl.dk, wl.dv, wl.chunk, dt_code)
        nseg = n2 if n2 > 0 else gdr.gdr_chunk_fwd_split_segments(wl.B, wl.H, wl.T, wl.dk, wl.dv, wl.chunk,
                                                                   dt_code)
        ws = None
        if n2 > 0:
            ws = torch.empty(gdr.gdr_chunk_fwd_two_phase_workspace(wl.B, wl.H, wl.T, wl.dk, wl.dv, wl.chunk, n2),
                             dtype=torch.uint8, device=dev)
        elif nseg > 1:
            ws = torch.empty(gdr.gdr_chunk_fwd_split_workspace(wl.B, wl.H, wl.dk, wl.dv, nseg),
                             dtype=torch.uint8, device=dev)

        def fwd():
            if n2 > 0:
                gdr.chunk_fwd_two_phase(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"],
                                        mode=mode, chunk=wl.chunk, nseg=n2, workspace=ws, o=o, S_T=ST)
            elif nseg > 1:
                gdr.chunk_fwd_split(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"],
                                    mode=mode, chunk=wl.chunk, nseg=nseg, workspace=ws, o=o, S_T=ST)
            else:
                gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["S0"], mode=mode,
                              chunk=wl.chunk, o=o, S_T=ST)

        def step():
            if flush is not None:
                flush.zero_()
            fwd()
        # one step = the whole forward, the unit of the roofline: with a sequence split three
        # launches (state pass, combine, output pass); the two-phase forward is phase one (two
        # launches, after a memset of its list count) and one state pass, or three with a split
        if n2 > 0:
            launches = 2 + (3 if n2 > 1 else 1)
            kern = (f"gdr wy_prep_kernel + wy_exact_kernel + state_pass_kernel"
                    + (f" x2 + split_combine_kernel (two-phase, {n2} segments)" if n2 > 1 else " (two-phase)"))
        else:
            launches = 3 if nseg > 1 else 1
            kern = kernel_name(wl, mode) if nseg <= 1 else \
                f"gdr chunk_tc_kernel x2 + split_combine_kernel (sequence split, {nseg} segments)"
        r.update(fwd=fwd, step=step, flush=flush, units=wl.units, bytes_per_launch=chunk_bytes(wl, mode),
                 launches_per_step=launches, flops=chunk_flops(wl), nseg=nseg, inp=inp,
                 out=(o, ST), kernel=kern, two_phase=n2 > 0)
    return r


def time_device(r, steps, warmup, world, local, stream):
    """W untimed steps, then `steps` timed ones: CUDA events on the launching stream around
    each step's launches (the L2 flush, if any, between them), clocks sampled meanwhile,
    barrier + synchronize on both sides.  Returns (mean ms per step, total ms, clocks)."""
    import linear_attention_recurrence_wy_b200 as gdr
    dev = torch.device("cuda", local)
    for _ in range(warmup):
        r["step"]()
    torch.cuda.synchronize(dev)
    rc = gdr.gdr_last_device_error(stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"device error after warm-up: {gdr.gdr_status_string(rc)}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(steps):
            if r["flush"] is not None:
                r["flush"].zero_()
            ev[i][0].record(stream)
            r["fwd"]()
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    rc = gdr.gdr_last_device_error(stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"device error in timed region: {gdr.gdr_status_string(rc)}")
    return sum(step_ms) / len(step_ms), t_start.elapsed_time(t_end), clk.summary()


def roofline_of(r, ms, hbm, tf_burst, peak_src):
    achieved = r["bytes_per_launch"] / (ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": traffic_for(r["name"], r["kernel"]), "peak_source": f"{peak_src} hbm_gbs",
            "kernel": r["kernel"]}
    if r["flops"] is not None:
        roof["tensor_context"] = {"flops_per_launch": r["flops"],
                                  "achieved_tflops": r["flops"] / (ms * 1e-3) / 1e12,
                                  "peak_tflops": tf_burst,
                                  "frac": r["flops"] / (ms * 1e-3) / 1e12 / tf_burst}
    return roof


# Workloads timed beside the headline on a one-GPU run (the `secondary` object): the decode
# target, the other chunked shapes, the fused token mixer and the backward.
SECONDARY = ("decode", "gdn_t2k", "gdn2_t16k", "gdn2_t16k_kda", "mixer_t4k", "bwd_t4k")


def run_secondary(names, steps, local, stream, hbm, tf_burst, peak_src):
    out = {}
    dev = torch.device("cuda", local)
    for name in names:
        r = setup_workload(name, 0, dev)
        ms, _, clk = time_device(r, steps, 3, 1, local, stream)
        n = steps
        if ms * steps < 250.0:
            # a timed region of at least ~0.25 s, so that the clock samples (every 100 ms) fall
            # inside it: the short workloads are timed again over more steps
            n = min(5000, math.ceil(250.0 / max(ms, 1e-3)))
            ms, _, clk = time_device(r, n, 3, 1, local, stream)
        roof = roofline_of(r, ms / (r["launches_per_step"] if name == "decode" else 1), hbm, tf_burst, peak_src)
        out[name] = {"ms_per_step": ms, "value": r["units"] / (ms * 1e-3), "unit": r["unit"],
                     "steps": n, "launches_per_step": r["launches_per_step"],
                     "config": config_of(name, 1), "roofline": roof, "clocks": clk}
        if name == "decode":
            out[name]["us_per_decode_step"] = 1e3 * ms / r["launches_per_step"]
        del r
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local):
    import linear_attention_recurrence_wy_b200 as gdr
    gdr.lib()
    name = args.workload
    dev = torch.device("cuda", local)
    hbm, tf_burst, tf_sust, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    r = setup_workload(name, rank, dev, decode_steps=args.decode_steps)
    wl, mode, units, unit = r["wl"], r["mode"], r["units"], r["unit"]
    kern_ms, total_ms, clk = time_device(r, args.steps, args.warmup, world, local, stream)
    ms_per_step = max_over_ranks(kern_ms, world)
    value = units * world / (ms_per_step * 1e-3)

    # end to end through the public API with host buffers (pinned), copies inside
    e2e = None
    if not args.no_e2e and name == "bwd_t4k":
        inp = r["inp"]
        hin = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in inp.items()}
        dOh, dSTh = r["dO"].cpu().pin_memory(), r["dST"].cpu().pin_memory()
        outh = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in r["grads"].items()}
        h2d = sum(v.numel() * v.element_size() for v in hin.values() if torch.is_tensor(v)) + \
            dOh.numel() * dOh.element_size() + dSTh.numel() * dSTh.element_size()
        d2h = sum(x.numel() * x.element_size() for x in outh.values())
        n_e2e = max(1, min(args.steps, 3))
        ws = r["ws"]

        def call():
            x = {k: (v.to(dev, non_blocking=True) if torch.is_tensor(v) else v) for k, v in hin.items()}
            g_ = gdr.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"],
                               dOh.to(dev, non_blocking=True), dSTh.to(dev, non_blocking=True), mode=mode,
                               workspace=ws)
            for k_, v_ in g_.items():
                outh[k_].copy_(v_, non_blocking=True)
        call()
        torch.cuda.synchronize(dev)
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            call()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world)
        e2e = {"value": units * world / (e2e_ms * 1e-3), "unit": unit,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
    elif not args.no_e2e and name == "mixer_t4k":
        c = wl
        inp = r["inp"]
        hin = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in inp.items()}
        h2d = sum(v.numel() * v.element_size() for v in hin.values() if torch.is_tensor(v))
        y, ST = r["out"]
        outh = (torch.empty(y.shape, dtype=y.dtype, pin_memory=True),
                torch.empty(ST.shape, dtype=ST.dtype, pin_memory=True))
        d2h = sum(x.numel() * x.element_size() for x in outh)
        n_e2e = max(1, min(args.steps, 5))
        call = lambda: gdr.mixer_fwd_host(hin["q"], hin["k"], hin["v"], hin["xg"], hin["xb"], hin["xw"],
                                          hin["z"], hin["weight"], hin["S0"], mode=c["mode"],
                                          layout=c["layout"], device=dev, out=outh)
        call()
        torch.cuda.synchronize(dev)
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            call()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world)
        e2e = {"value": units * world / (e2e_ms * 1e-3), "unit": unit,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
    elif not args.no_e2e and name != "decode":
        inp = r["inp"]
        hin = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in inp.items()}
        h2d = sum(v.numel() * v.element_size() for v in hin.values() if torch.is_tensor(v))
        o, ST = r["out"]
        outh = (torch.empty(o.shape, dtype=o.dtype, pin_memory=True),
                torch.empty(ST.shape, dtype=ST.dtype, pin_memory=True))
        d2h = sum(x.numel() * x.element_size() for x in outh)
        n_e2e = max(1, min(args.steps, 5))
        call = lambda: gdr.chunk_fwd_host(hin["q"], hin["k"], hin["v"], hin["g"], hin["b"], hin["w"],
                                          hin["S0"], mode=mode, chunk=wl.chunk, device=dev, out=outh)
        call()
        torch.cuda.synchronize(dev)
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            call()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world)
        e2e = {"value": units * world / (e2e_ms * 1e-3), "unit": unit,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    launches_per_step = r["launches_per_step"]
    # the roofline's unit: one decode launch, else the whole step
    launch_ms = kern_ms / launches_per_step if name == "decode" else kern_ms
    roof = roofline_of(r, launch_ms, hbm, tf_burst, peak_src)
    del r
    torch.cuda.empty_cache()
    secondary = None
    if world == 1 and not args.no_secondary and BATCH is None:
        secondary = run_secondary([n for n in SECONDARY if n != name], args.secondary_steps, local, stream,
                                  hbm, tf_burst, peak_src)
    if rank != 0:
        return
    line = {"metric": metric_name(name), "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if (name in ("decode", "mixer_t4k", "bwd_t4k") or wl.dtype == "bf16") else "f32",
            "data": "synthetic", "config": config_of(name, world), "roofline": roof,
            "clocks": clk, "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e, "wall_total_ms": total_ms}
    if name != "decode":
        # the same throughput for a whole layer of H heads: B*T / step time
        line["layer_tokens_per_s"] = value / (wl["H"] if name == "mixer_t4k" else wl.H)
    if secondary is not None:
        line["secondary"] = secondary
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(name, target_cpu_s=args.ref_cpu_s)
    print(json.dumps(line), flush=True)


# ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant kernel,
# keyed by workload and by a digest of the kernel's sources at capture time (a changed
# kernel reports null until it is captured again); see profiles/.
TRAFFIC = {
    ("gdn2_t4k", "chunk_tc"): (949.304064e6 + 124.721920e6, "09a47ac0"),
    ("decode", "decode"): (275.801088e6 + 210.006784e6, "e0c71d93"),
    ("mixer_t4k", "chunk_tc"): (1129.626368e6 + 125.486080e6, "09a47ac0"),
    # the backward's step (its four launches: checkpoints, state gradient, per-chunk
    # gradients, the strong-decay list), captured one kernel at a time on one sequence of
    # the workload and scaled by the 8 sequences: the inputs are read by three launches
    ("bwd_t4k", "bwd"): (8 * (422.868992e6 + 112.833024e6), "f113754a"),
    # the two-phase forward's step (phase one, the exact-path kernel, the state pass or its
    # split's two passes and the chaining kernel), one kernel per capture: the records add
    # their write and read to the inputs and the output
    ("gdn2_t16k", "two_phase"): (972.075008e6 + 313.840128e6, "3a0deb3e"),
    ("gdn_t2k", "two_phase"): (253.977856e6 + 115.448832e6, "3a0deb3e"),
}


def _src_digest(files):
    import hashlib
    h = hashlib.sha1()
    for f in files:
        h.update(open(os.path.join(ROOT, "linear_attention_recurrence_wy_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:8]


def traffic_for(name, kname):
    if BATCH is not None:
        return None   # the recorded figures are for the workloads' own sizes
    if name == "decode":
        key, files = ("decode", "decode"), ["decode.cu"]
    elif name == "bwd_t4k":
        key, files = ("bwd_t4k", "bwd"), ["chunk_tc.cu", "tri_inverse.cuh", "tc_util.cuh", "bwd_tc.cu", "bwd.cu"]
    elif "two-phase" in kname:
        key, files = (name, "two_phase"), ["wy_prep.cu", "state_pass.cu", "split.cu", "two_phase.cuh",
                                           "tri_inverse.cuh", "tc_util.cuh"]
    elif "chunk_tc" in kname and "split" not in kname:
        key, files = (name, "chunk_tc"), ["chunk_tc.cu", "tri_inverse.cuh", "tc_util.cuh"]
    else:
        return None
    rec = TRAFFIC.get(key)
    if rec is None:
        return None
    value, digest = rec
    return value if _src_digest(files) == digest else None


def kernel_name(wl, mode):
    if wl.dtype == "bf16" and wl.dk == 128 and wl.dv == 128 and wl.chunk == 64:
        return "gdr chunk_tc_kernel (tcgen05)"
    return "gdr chunk_simt_kernel"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gdn2_t4k",
                    choices=["gdn2_t4k", "gdn_t2k", "gdn2_t16k", "gdn2_t16k_kda", "gdn2_tiny", "decode",
                             "gdn2_t4k_bonly", "gdn2_t4k_wonly", "mixer_t4k", "bwd_t4k"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads timed beside the headline on a one-GPU run")
    ap.add_argument("--secondary-steps", type=int, default=10)
    ap.add_argument("--ref-cpu-s", type=float, default=15.0)
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="decode steps per bench step (default: the workload's 1000); fewer keep an "
                         "ncu capture's launch count small")
    ap.add_argument("--batch", type=int, default=None,
                    help="run B sequences instead of the workload's own (chunked forward and backward "
                         "workloads): a small case for ncu captures")
    args = ap.parse_args()
    global BATCH
    BATCH = args.batch
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
