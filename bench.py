"""Benchmark of the POET-X linear layer step (CNP rebuild + forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload KEY] [--tokens T]
                    [--impl ours|reference] [--xq | --xq-staged] [--first-linear-only]

One step is the whole hot path over one batch, for every linear of the workload: poetx_cnp_build
for R and P (where the workload's step includes it), poetx_linear_fwd, poetx_linear_bwd (dx, dq_r,
dq_p), and merge_reinit amortised over its period where the workload has one.  Inputs are synthetic
(seeded, poetx_workloads) and resident in HBM before the timed region.  --xq stores W0' in 8 bits
(int8 codes + column scales, dequantised inside the W0' products); --xq-staged dequantises it
into the workspace once per product instead.  For N > 1 (torchrun, one rank per GPU) every rank runs the step
on its own tokens (weak scaling) and the packed dq gradients are summed over ranks with NCCL,
as data-parallel training does.  Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle on the host cores instead (a bounded sample of the
same workload per step); under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import poetx_workloads as W  # noqa: E402

METRIC = "POET-X linear fwd+bwd tokens/s at Llama-8B shapes; % of 1-B200 roofline"
DEFAULT_WORKLOAD = "llama8b_up_proj"
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- helpers
def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_tag() -> str:
    """First 12 hex digits of the SHA-256 of the tensor-core GEMM source: DRAM traffic figures
    taken with ncu are used only while the kernel is the one they were taken on."""
    import hashlib
    src = os.path.join(ROOT, "orthogonal_equivalence_build_b200", "csrc", "umma_gemm.cu")
    return hashlib.sha256(open(src, "rb").read()).hexdigest()[:12]


def measured_traffic(names, T):
    """Mean dram__bytes_read.sum + dram__bytes_write.sum per launch of the kernels `names` at T
    tokens, from profiles/traffic.txt (lines "<kernel> <T> <bytes per launch> <source tag>"),
    or None when there is no figure for this kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    tag, vals = kernel_source_tag(), []
    for ln in open(path):
        parts = ln.split()
        if (len(parts) == 4 and parts[0] in names and parts[1] == str(T) and parts[3] == tag):
            vals.append(float(parts[2]))
    return sum(vals) / len(vals) if vals else None


def layer_flops(T, m, n, b, cnp=True):
    """Algorithmic FLOPs of one step: fwd 2T(mb+mn+nb), bwd dx 2T(mn+mb+nb), dG 2T(mb+nb),
    CNP 2 products per block (S = QQ and S(2I+2Q+S)), dq 4 products per block."""
    f = 2 * T * (m * b + m * n + n * b) * 2 + 2 * T * (m * b + n * b)
    nblk = m // b + n // b
    if cnp:
        f += nblk * (2 * 2 * b ** 3 + 4 * 2 * b ** 3)
    return f


def layer_bytes(T, m, n, b, e=2, w_e=None):
    """Algorithmic HBM bytes of one step: boundary tensors plus the saved activations.
    fwd reads X, W0', G and writes Y, B and A = X[:, perm_r]; bwd reads dY, A, B, W0', G and
    writes dX; q, G, dq in fp32.  w_e: bytes per W0' element (1 for 8-bit storage, plus its
    column scales)."""
    gblk = (m // b + n // b) * b * b
    qn = (m // b + n // b) * b * (b - 1) // 2
    w = (e if w_e is None else w_e) * m * n + (4 * n if w_e == 1 else 0)
    fwd = e * (T * m + T * n + T * n + T * m) + w + e * gblk
    bwd = e * (T * n + T * m + T * n + T * m) + w + e * gblk
    cnp = 4 * qn + 4 * gblk + 2 * gblk
    dq = 4 * qn * 2
    return fwd + bwd + cnp + dq


def sum_over_ranks_(flat, group=None):
    """Data-parallel reduction of the packed dq gradients: dq is linear in dG, and dG is a sum
    over tokens, so the dq of the whole batch is the sum of the ranks' dq."""
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat


class DqReducer:
    """Data-parallel sum of the packed dq gradients, one asynchronous all-reduce per linear,
    issued as soon as that linear's backward is enqueued: the collective then runs on the
    communicator's own stream while the next linear's kernels run, and finish() makes the
    caller's stream (NCCL) or the caller (gloo) wait for all of them before the step ends. Every
    rank issues the same collectives in the same order: linear 0, 1, ...  With one rank it does
    nothing."""

    def __init__(self, group=None):
        self.group = group
        self.works = []

    def add(self, flat):
        import torch.distributed as dist
        if dist.is_initialized() and dist.get_world_size(self.group) > 1:
            self.works.append(dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=self.group,
                                              async_op=True))

    def finish(self):
        for w in self.works:
            w.wait()
        self.works.clear()


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The job's time is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_initialized() and dist.get_world_size(group) > 1):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


class ClockSampler:
    """SM clock and clock-event reasons sampled every 5 ms through NVML (read-only queries)
    while the timed region runs."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, torch_device: int):
        self.dev = torch_device
        self.samples = []
        self.reasons = set()
        self.smax = 0.0
        self._stop = threading.Event()
        self.t = None
        self.nv = None

    def _handle(self):
        import pynvml as nv
        import torch
        nv.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return nv, nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            return nv, nv.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        try:
            self.nv, self.h = self._handle()
            self.smax = float(self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        except Exception:
            self.nv = None
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS:
                    bit = getattr(nv, attr, 0)
                    if bit and mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.005)

    def stop(self):
        if self.t is None:
            return None
        self._stop.set()
        self.t.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.smax,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "NVML, 5 ms period, timed region only"}


# ----------------------------------------------------------------------------- oracle arm
_SAMPLE_CACHE = {}


def oracle_step_sample(wl, T_sample: int, nlin: int = 1):
    """One float64 oracle step (CNP of R and P, forward, backward with dq) of the workload's
    first nlin linears on T_sample tokens.  Returns (seconds, tokens)."""
    import oracle as O
    key = (wl.key, T_sample, nlin)
    if key not in _SAMPLE_CACHE:
        items = []
        for li in range(nlin):
            p = W.layer_params(wl, li)
            a = W.layer_acts(wl, li, tokens=T_sample)
            items.append((p, a, O.merge_permutations(p["W0"], p["perm_r"], p["perm_p"])))
        _SAMPLE_CACHE[key] = items
    t0 = time.perf_counter()
    for p, a, W0m in _SAMPLE_CACHE[key]:
        G_r, G_p = O.cnp(p["q_r"], wl.b), O.cnp(p["q_p"], wl.b)
        O.linear_bwd(a["X"], a["dY"], W0m, p["perm_r"], p["perm_p"], G_r, G_p, p["q_r"],
                     p["q_p"], wl.b)
    return time.perf_counter() - t0, T_sample


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def blas_name():
    try:
        from threadpoolctl import threadpool_info
        for d in threadpool_info():
            if d.get("user_api") == "blas":
                return f"{d.get('internal_api')} {d.get('version')}"
    except Exception:
        pass
    return "unknown"


def sample_text(wl, T_sample, nlin):
    what = f"the {wl.key} layer" if nlin == 1 else f"the {nlin} linears of {wl.key}"
    return (f"one float64 oracle step (CNP + fwd + bwd with dq) of {what} on {T_sample} of its "
            f"{wl.tokens} tokens")


def oracle_merge_sample(wl, nlin, T_sample):
    """Seconds of one float64 oracle merge_reinit of the workload's first nlin linears (the
    layers cached by oracle_step_sample)."""
    import oracle as O
    items = _SAMPLE_CACHE[(wl.key, T_sample, nlin)]
    t0 = time.perf_counter()
    for p, _, W0m in items:
        O.merge_reinit(W0m, p["perm_r"], p["perm_p"], p["q_r"], p["q_p"], wl.b, 0x5EED)
    return time.perf_counter() - t0


def cpu_baseline(wl, T_sample, nlin=1):
    """The oracle as it stands on a bounded sample, on every BLAS thread; plus the same sample
    of the first linear on one thread, and for a workload with a merge period one merge_reinit
    spread over that period (an extrapolation, labelled as one)."""
    dt, tok = oracle_step_sample(wl, T_sample, nlin)
    out = {"value": tok / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"{sample_text(wl, T_sample, nlin)}: {dt:.2f} s", "blas": blas_name(),
           "seconds": dt}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"):
            dt1, _ = oracle_step_sample(wl, T_sample, 1)
        out["one_thread"] = {"value": T_sample / dt1, "unit": "tokens/s",
                             "sample": f"{sample_text(wl, T_sample, 1)} on 1 BLAS thread: "
                                       f"{dt1:.2f} s"}
    except Exception as e:   # threadpoolctl missing: report why
        out["one_thread"] = {"unavailable": str(e)}
    if wl.merge_every:
        dm = oracle_merge_sample(wl, nlin, T_sample)
        per_step = dt + dm / wl.merge_every
        out["extrapolated_with_merge"] = {
            "value": T_sample / per_step, "unit": "tokens/s", "merge_reinit_s": dm,
            "label": (f"extrapolated, not run for {wl.merge_every} steps: the sampled step plus "
                      f"one oracle merge_reinit of the {nlin} linears ({dm:.2f} s) spread over "
                      f"its {wl.merge_every}-step period")}
    return out


def workload_config(wl, args, world):
    """The `config` object of the JSON line, the same for both arms: the workload as run (its
    linears, block size, tokens, parallelism, what one step holds, how L2 is kept cold)."""
    T = args.tokens or wl.tokens
    esz = 2 if wl.dtype == "bf16" else 4
    lins = wl.linears if args.all_linears else wl.linears[:1]
    in_bytes = sum(T * (lin.m + lin.n) * esz for lin in lins)
    cfg = {"workload": wl.key, "linears": [f"{lin.name} {lin.m}x{lin.n}" for lin in lins],
           "b": wl.b, "tokens_per_gpu": T, "global_batch_tokens": T * world,
           "parallelism": f"dp{world}",
           "step": (("cnp_build(R,P) of all linears in one call + " if len(lins) > 1
                     else "cnp_build(R,P) + ") if wl.cnp_in_step else "")
           + ("linear_fwd + linear_bwd(dx, dq) per linear" if len(lins) == 1 else
              "linear_fwd + linear_bwd_dg(dx, dG) per linear + dq of all linears in one call")
           + (", activation A = X[:, perm_r] [T, m] kept from forward to backward, B [T, n] "
              "rebuilt in the backward" if getattr(args, "xmem", False) else
              ", activations B [T, n] and A = X[:, perm_r] [T, m] kept from forward to backward")
           + (" + NCCL all-reduce of dq" if world > 1 else ""),
           "l2": (f"inputs larger than L2: X + dY = {in_bytes / 2**20:.0f} MiB per step"
                  if in_bytes > L2_BYTES else "L2 flushed (2x126 MiB write) between steps")}
    if len(lins) == 1:
        cfg.update({"m": lins[0].m, "n": lins[0].n})
    if args.xq:
        cfg["w0m_storage"] = (
            "int8 codes + fp32 column scales, dequantised to bf16 "
            + ("into the workspace once per W0' product (staged)" if args.xq_staged
               else "in the W0' GEMMs' shared-memory operand stages"))
    if getattr(args, "xmem", False):
        cfg["saved_b"] = ("none (POET-Xmem): the backward rebuilds B = A' W0' from the kept A; "
                          "the roofline counts the forward work only")
    if getattr(args, "fuse_w0p", False):
        cfg["fused_w0_p"] = "forward W0' product and P-block product in one kernel"
    if wl.merge_every:
        cfg["merge_reinit"] = f"every {wl.merge_every} steps, amortised into ms_per_step"
    return cfg


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    wl = W.WORKLOADS[args.workload]
    nlin = len(wl.linears) if args.all_linears else 1
    T_sample = args.ref_tokens
    times = []
    for i in range(args.warmup + args.steps):
        dt, _ = oracle_step_sample(wl, T_sample, nlin)
        if i >= args.warmup:
            times.append(dt)
    sec = statistics.mean(times)
    value = T_sample / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "blas": blas_name(),
                         "sample": sample_text(wl, T_sample, nlin)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from orthogonal_equivalence_build_b200 import poetx

    rank, local, world = env_rank()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl = W.WORKLOADS[args.workload]
    b = wl.b
    T = args.tokens or wl.tokens
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    esz = 2 if dt == torch.bfloat16 else 4
    nlin = len(wl.linears) if args.all_linears else 1

    # ---- every linear of the workload (the same layers on every rank, each rank its own tokens)
    layers = []
    for li in range(nlin):
        lin = wl.linears[li]
        p = W.layer_params(wl, li)
        a = W.layer_acts(wl, li, tokens=T, seed=W.WORKLOAD_SEED[wl.key] * 1000 + rank)
        w0 = torch.from_numpy(p["W0"]).to(dt).to(dev)
        pr = torch.from_numpy(p["perm_r"]).to(dev)
        pp = torch.from_numpy(p["perm_p"]).to(dev)
        w0m = torch.empty_like(w0)
        poetx.merge_permutations(w0, pr, pp, w0m)
        del w0
        scale = None
        if args.xq:   # 8-bit W0' (int8 codes + fp32 column scales)
            wq = torch.empty(w0m.shape, dtype=torch.int8, device=dev)
            scale = torch.empty(w0m.shape[1], dtype=torch.float32, device=dev)
            poetx.quantize_w0(w0m, wq, scale)
            w0m = wq
        L = poetx.PoetxLinear(w0m, pr, pp, torch.from_numpy(p["q_r"]).to(dev),
                              torch.from_numpy(p["q_p"]).to(dev), b, w0m_scale=scale,
                              staged=args.xq_staged, fused_w0_p=args.fuse_w0p)
        d = {"lin": lin, "layer": L,
             "x_host": torch.from_numpy(a["X"]).to(dt).pin_memory(),
             "dy_host": torch.from_numpy(a["dY"]).to(dt).pin_memory()}
        del a
        d["x"] = d["x_host"].to(dev)
        d["dy"] = d["dy_host"].to(dev)
        d["y"] = torch.empty(T, lin.n, dtype=dt, device=dev)
        # activations kept from the forward for the backward: B (POET-Xfast; with --xmem it is
        # not kept and the backward rebuilds it, POET-Xmem), and A = X[:, perm_r]
        d["bsave"] = None if args.xmem else torch.empty(T, lin.n, dtype=dt, device=dev)
        d["asave"] = torch.empty(T, lin.m, dtype=dt, device=dev)
        if nlin > 1:   # per-block gradients, for one dq pass over every linear
            d["dG"] = torch.empty(lin.m // b + lin.n // b, b, b, device=dev)
        d["dx"] = torch.empty(T, lin.m, dtype=dt, device=dev)
        # dq_r and dq_p are views of one packed buffer: one all-reduce per linear (N > 1)
        d["dq"] = torch.empty(L.q_r.numel() + L.q_p.numel(), device=dev)
        d["dq_r"] = d["dq"][:L.q_r.numel()].view_as(L.q_r)
        d["dq_p"] = d["dq"][L.q_r.numel():].view_as(L.q_p)
        layers.append(d)
        poetx.layer_cnp_build(L)
    all_layers = [d["layer"] for d in layers]
    ws = torch.empty(max(max(max(poetx.fwd_workspace_bytes(d["layer"], T),
                                 poetx.bwd_workspace_bytes(d["layer"], T)) for d in layers),
                         poetx.layers_cnp_workspace_bytes(all_layers),
                         poetx.layers_dq_workspace_bytes(all_layers)),
                     dtype=torch.uint8, device=dev)
    reducer = DqReducer()
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum((d["x"].numel() + d["dy"].numel()) * esz for d in layers)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if in_bytes <= L2_BYTES else None

    def step(xs=None, dys=None, outs=None):
        """One step over every linear; outs[i] = (y, dx, dq) of linear i, dq the packed
        [dq_r, dq_p] (default: the layer's own result buffers). One linear: its backward forms
        dq. Several: each backward stops at the per-block gradients dG and one call forms every
        linear's dq (more blocks per launch). With N > 1 each linear's dq is summed over the
        ranks by an all-reduce issued as soon as it exists, overlapping the kernels after it."""
        if wl.cnp_in_step:
            # every linear's CNP blocks in one call (one layer: poetx_layer_cnp_build's work)
            poetx.layers_cnp_build(all_layers, ws)
        dqs = []
        for i, d in enumerate(layers):
            L = d["layer"]
            xin = d["x"] if xs is None else xs[i]
            dyin = d["dy"] if dys is None else dys[i]
            y, dx, dq = (d["y"], d["dx"], d["dq"]) if outs is None else outs[i]
            dqs.append(dq)
            nr = L.q_r.numel()
            poetx.linear_fwd(L, xin, y, d["bsave"], ws, saved_a=d["asave"])
            if nlin == 1:
                poetx.linear_bwd(L, xin, dyin, d["bsave"], dx, dq[:nr].view_as(L.q_r),
                                 dq[nr:].view_as(L.q_p), ws, saved_a=d["asave"])
                reducer.add(dq)
            else:
                poetx.linear_bwd_dg(L, xin, dyin, d["bsave"], dx, d["dG"], ws,
                                    saved_a=d["asave"])
        if nlin > 1:
            poetx.layers_dq_from_dg(all_layers, [d["dG"] for d in layers],
                                    [dq[:d["layer"].q_r.numel()] for d, dq in zip(layers, dqs)],
                                    [dq[d["layer"].q_r.numel():] for d, dq in zip(layers, dqs)],
                                    ws)
            for dq in dqs:
                reducer.add(dq)
        reducer.finish()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    poetx.device_status()

    # ---- timed region (device time, per-step CUDA events, kernel trace on)
    sampler = ClockSampler(local)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    # events only around the dominant kernel inside the timed region: an event between two
    # launches keeps the second from overlapping the first one's tail
    # (with --xmem the backward's rebuild of B is a third W0' product, "umma_dense_W0")
    w0_names = (("umma_dense_W0_i8", "umma_dense_W0T_i8") if args.xq and not args.xq_staged
                else ("umma_w0p_fused", "umma_dense_W0T", "umma_dense_W0") if args.fuse_w0p
                else ("umma_dense_W0", "umma_dense_W0T"))
    poetx.trace_read()
    poetx.trace_select(w0_names)
    poetx.trace_enable(True)
    sampler.start()
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    poetx.trace_enable(False)
    trace = poetx.trace_read()
    step_ms_local = sum(s.elapsed_time(e) for s, e in ev) / args.steps

    # ---- merge-then-reinitialize, when the workload's schedule has it (amortised per step)
    merge_ms = 0.0
    if wl.merge_every:
        # the workspace is allocated before the timed region, as a training loop would keep it
        mws = torch.empty(max(poetx.merge_reinit_workspace_bytes(d["layer"]) for d in layers),
                          dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for d in layers:
            poetx.merge_reinit(d["layer"], 0x5EED + rank, workspace=mws)
        e1.record(stream)
        torch.cuda.synchronize()
        merge_ms = e0.elapsed_time(e1)
        for d in layers:   # restore a non-trivial q for any later use
            poetx.layer_cnp_build(d["layer"])
    step_ms_local += merge_ms / max(wl.merge_every, 1) if wl.merge_every else 0.0
    ms_per_step = max_over_ranks(step_ms_local, dev)
    value = T * world / (ms_per_step / 1e3)

    # ---- dominant kernel: the W0' GEMMs of all linears
    w0_ms = [ms for name, ms in trace if name in w0_names]
    # every library launch of a step, with its device time: a separate traced pass (3 steps)
    poetx.trace_select(None)
    poetx.trace_enable(True)
    n_pass = 3
    for _ in range(n_pass):
        step()
    torch.cuda.synchronize()
    poetx.trace_enable(False)
    full = poetx.trace_read()
    launches = len(full) // n_pass * args.steps
    per_kernel = {}
    for name, ms in full:
        per_kernel[name] = per_kernel.get(name, 0.0) + ms / n_pass
    peaks, peak_src = measured_peaks()
    roofline = None
    if w0_ms:
        # (the fused forward kernel also does the P-block product: 2 T n b more)
        flops = sum(2.0 * (3 if args.xmem else 2) * T * d["lin"].m * d["lin"].n
                    + (2.0 * T * d["lin"].n * b if args.fuse_w0p else 0.0)
                    for d in layers) * args.steps
        total_ms = sum(w0_ms)
        achieved = flops / (total_ms / 1e3) / 1e12
        # The W0' products are timed inside a sub-second region at the clock the bench samples,
        # so the denominator is the burst figure (a cuBLAS bf16 GEMM timed alone). The sustained
        # figure comes from a seconds-long loop that settles at a much lower clock under the
        # power cap; its ratio is kept only as a labelled aside.
        peak = peaks["bf16_tflops"]
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "kernel": f"{w0_names[0]} / {w0_names[1]} (B = A' W0'"
                              + (" with C = B Diag(G_P)" if args.fuse_w0p else "")
                              + ", dA' = dB W0'^T)",
                    "peak_source": f"{peak_src} bf16_tflops (burst)",
                    "aside_frac_of_sustained_peak": (
                        achieved / peaks["bf16_tflops_sustained"]
                        if "bf16_tflops_sustained" in peaks else None),
                    "avg_launch_ms": total_ms / len(w0_ms), "launches": len(w0_ms)}
        if nlin == 1 and not args.fuse_w0p and not args.xmem:
            roofline["traffic"] = measured_traffic(w0_names, T)
    F = sum(layer_flops(T, d["lin"].m, d["lin"].n, b, wl.cnp_in_step) for d in layers)
    Bb = sum(layer_bytes(T, d["lin"].m, d["lin"].n, b, esz, 1 if args.xq else None)
             for d in layers)
    t_roof = max(F / (peaks["bf16_tflops"] * 1e12), Bb / (peaks["hbm_gbs"] * 1e9))

    # ---- end to end through the API: pinned host inputs in, every result out (Y, dX, dq_r,
    # dq_p of every linear), every step. Inputs and outputs are double-buffered on the device:
    # the upload of step i+1's X and dY (one copy stream) and the download of step i-1's
    # results (another copy stream) overlap step i's kernels. A step starts when its inputs
    # have landed and the download that last read its output set has finished; an upload
    # starts when the step that last read its input buffer has finished. The timed region ends
    # after the last step's results are in host memory.
    out_host = [(torch.empty(T, d["lin"].n, dtype=dt).pin_memory(),
                 torch.empty(T, d["lin"].m, dtype=dt).pin_memory(),
                 torch.empty(d["dq"].shape, dtype=torch.float32).pin_memory())
                for d in layers]
    bufs = [([torch.empty_like(d["x"]) for d in layers], [torch.empty_like(d["dy"]) for d in layers])
            for _ in range(2)]
    outs = [[(d["y"], d["dx"], d["dq"]) if k == 0 else
             (torch.empty_like(d["y"]), torch.empty_like(d["dx"]), torch.empty_like(d["dq"]))
             for d in layers] for k in range(2)]
    h2d_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(3, min(args.steps, 6))
    d2h_bytes = sum(t.numel() * t.element_size() for o in out_host for t in o)

    def upload(k):
        h2d_stream.wait_event(consumed[k])
        with torch.cuda.stream(h2d_stream):
            for i, d in enumerate(layers):
                bufs[k][0][i].copy_(d["x_host"], non_blocking=True)
                bufs[k][1][i].copy_(d["dy_host"], non_blocking=True)
        copied[k].record(h2d_stream)

    def download(k):
        d2h_stream.wait_event(computed[k])
        with torch.cuda.stream(d2h_stream):
            for i in range(len(layers)):
                for host, dev_t in zip(out_host[i], outs[k][i]):
                    host.copy_(dev_t, non_blocking=True)
        downloaded[k].record(d2h_stream)

    def run_step(k):
        stream.wait_event(copied[k])
        stream.wait_event(downloaded[k])
        step(bufs[k][0], bufs[k][1], outs[k])
        consumed[k].record(stream)
        computed[k].record(stream)
        download(k)

    def e2e_run(n):
        h2d_stream.wait_stream(stream)
        d2h_stream.wait_stream(stream)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload((i + 1) % 2)
            run_step(i % 2)
        stream.wait_stream(d2h_stream)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e = {"value": T * world * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": d2h_bytes,
           "returned": "Y, dX, dq_r, dq_p of every linear",
           "pipeline": ("inputs of step i+1 upload on one copy stream and results of step i-1 "
                        "download on another during step i")}

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(wl, args.ref_tokens, nlin)
            cpu.pop("seconds", None)
        cfg = workload_config(wl, args, world)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if dt == torch.bfloat16 else "f32", "data": "synthetic",
            "config": cfg,
            "tflops": F * world / (ms_per_step / 1e3) / 1e12,
            "step_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_per_step,
                              "flops": F, "bytes": Bb, "peaks": peak_src},
            "roofline": roofline,
            "cpu_baseline": cpu,
            **({"merge_reinit_ms": merge_ms} if wl.merge_every else {}),
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
            "kernel_ms_per_step": {k: v for k, v in sorted(per_kernel.items(),
                                                                        key=lambda kv: -kv[1])},
            "kernel_ms_source": ("CUDA events around every library launch, separate pass of "
                                 f"{n_pass} steps after the timed region (which records events "
                                 "around the W0' GEMMs only)"),
        }
        if (world == 1 and args.other_configs and args.workload == DEFAULT_WORKLOAD
                and not (args.xq or args.xmem or args.fuse_w0p or args.tokens)):
            line["other_configs"] = other_configs(args)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


OTHER_WORKLOADS = ("llama1p3b_attn", "llama8b_decoder", "llama13b_layers")


def other_configs(args):
    """The other bf16 workloads, each measured by this script in a process of its own after the
    headline run (same GPU, default steps unless fewer are asked): a summary of each one's line
    (its step time, tokens/s, step roofline fraction, W0' rate and clocks), so that one run of
    the benchmark reports every configuration. A workload that fails is reported as such."""
    import subprocess
    out = {}
    for key in OTHER_WORKLOADS:
        cmd = [sys.executable, os.path.abspath(__file__), "--workload", key, "--no-cpu-baseline",
               "--no-other-configs", "--steps", str(args.steps), "--warmup", str(args.warmup)]
        try:
            r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
            lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
            if r.returncode != 0 or not lines:
                out[key] = {"error": f"exit {r.returncode}: " + (r.stderr.strip().splitlines()
                                                                 or ["no output"])[-1][:200]}
                continue
            d = json.loads(lines[-1])
            rl = d.get("roofline") or {}
            out[key] = {"ms_per_step": d["ms_per_step"], "value": d["value"], "unit": d["unit"],
                        "steps": d["steps"], "step_roofline_frac": d["step_roofline"]["frac"],
                        "w0_tflops": rl.get("achieved"), "clocks": d.get("clocks"),
                        "e2e": (d.get("e2e") or {}).get("value"),
                        "linears": d["config"].get("linears")}
        except Exception as ex:   # a timeout or an unparsable line: reported, not fatal
            out[key] = {"error": f"{type(ex).__name__}: {ex}"[:200]}
    return out


def run_vs_cublas(args):
    """The library's tensor-core kernels against cuBLAS (torch.matmul / torch.bmm) on the same
    bf16 operands in the same process, at the workload's shapes: the block-diagonal product of
    the P side (all n/b blocks of the T-token activation, stacked as one [n/b * T, b] x [b, b]
    product, and as the strided batched form straight from the [T, n] activation) and the
    forward W0' product [T, m] x [m, n]. L2 is flushed before every timed launch; medians of
    --steps launches after --warmup. One JSON line; outputs are compared element by element."""
    import torch
    from orthogonal_equivalence_build_b200 import poetx
    wl = W.WORKLOADS[args.workload]
    m, n = wl.linears[0].m, wl.linears[0].n
    b, T = wl.b, args.tokens or wl.tokens
    nb = n // b
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def med_ms(fn):
        for _ in range(args.warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(c) for a, c in ev)

    g = torch.Generator(device="cuda").manual_seed(7)
    out = {"mode": "vs_cublas", "workload": args.workload, "T": T, "m": m, "n": n, "b": b,
           "l2": "flushed before every launch", "steps": args.steps}
    # block-diagonal product: bytes read + written, FLOPs
    A = torch.randn(nb * T, b, device="cuda", generator=g).to(torch.bfloat16)
    G = (torch.randn(b, b, device="cuda", generator=g) * 0.05).to(torch.bfloat16)
    C, C2 = (torch.empty(nb * T, b, device="cuda", dtype=torch.bfloat16) for _ in range(2))
    byt, fl = 2.0 * nb * T * b * 2, 2.0 * nb * T * b * b
    rows = {}
    ms = med_ms(lambda: poetx.testing_gemm_bf16(A, False, G, True, nb * T, b, b, C, variant=1))
    rows["ours_block_stacked"] = ms
    ms = med_ms(lambda: torch.matmul(A, G, out=C2))
    rows["cublas_block_stacked"] = ms
    same_block = bool(torch.equal(C, C2))
    del A, C, C2
    X = torch.randn(T, n, device="cuda", generator=g).to(torch.bfloat16)
    Gb = (torch.randn(nb, b, b, device="cuda", generator=g) * 0.05).to(torch.bfloat16)
    Cb = torch.empty(nb, T, b, device="cuda", dtype=torch.bfloat16)
    Xv = X.view(T, nb, b).permute(1, 0, 2)
    rows["cublas_block_bmm_strided"] = med_ms(lambda: torch.bmm(Xv, Gb, out=Cb))
    del X, Gb, Cb
    for k in list(rows):
        ms = rows[k]
        rows[k] = {"ms": ms, "TB/s": byt / ms / 1e9, "TFLOP/s": fl / ms / 1e9}
    out["block_product"] = rows
    out["block_product_outputs_equal"] = same_block
    # forward W0' product
    Ap = torch.randn(T, m, device="cuda", generator=g).to(torch.bfloat16)
    W0 = (torch.randn(m, n, device="cuda", generator=g) * m ** -0.5).to(torch.bfloat16)
    B1, B2 = (torch.empty(T, n, device="cuda", dtype=torch.bfloat16) for _ in range(2))
    fl = 2.0 * T * m * n
    rows = {"ours_w0": med_ms(lambda: poetx.testing_gemm_bf16(Ap, False, W0, True, T, n, m, B1,
                                                             variant=2)),
            "cublas_w0": med_ms(lambda: torch.matmul(Ap, W0, out=B2))}
    out["w0_product"] = {k: {"ms": v, "TFLOP/s": fl / v / 1e9} for k, v in rows.items()}
    out["w0_outputs_max_rel_diff"] = float((B1.float() - B2.float()).abs().max()
                                           / B2.float().abs().max())
    poetx.device_status()
    print(json.dumps(out), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0, help="override tokens per GPU")
    ap.add_argument("--ref-tokens", type=int, default=256,
                    help="tokens in the oracle's bounded sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--first-linear-only", dest="all_linears", action="store_false",
                    help="time only the first linear of a multi-linear workload")
    ap.add_argument("--xq", action="store_true",
                    help="store W0' in 8 bits (int8 + column scales) and time that layer")
    ap.add_argument("--xq-staged", action="store_true",
                    help="with --xq: dequantise W0' into the workspace once per product")
    ap.add_argument("--no-other-configs", dest="other_configs", action="store_false",
                    help="with the default workload on one GPU, do not also run the other bf16 "
                         "workloads (each in a process of its own) for the other_configs key")
    ap.add_argument("--xmem", action="store_true",
                    help="keep no B from the forward (POET-Xmem): the backward rebuilds it")
    ap.add_argument("--fuse-w0p", action="store_true",
                    help="set POETX_LAYER_FUSED_W0_P on every linear (the forward's W0' and "
                         "P-block products in one kernel where it applies)")
    ap.add_argument("--vs-cublas", action="store_true",
                    help="time the block-diagonal and W0' products against cuBLAS on the same "
                         "operands (one GPU) and print that comparison instead")
    args = ap.parse_args(argv)
    if args.vs_cublas:
        return run_vs_cublas(args)
    if args.xq_staged:
        args.xq = True
    if args.warmup < 3 and args.impl == "ours" and not os.environ.get("POETX_BENCH_ALLOW_SHORT"):
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
