"""Benchmark of the calibration-free sparse routed-expert reader.

Workload (default): one Qwen3-30B-A3B-shaped MoE layer (d=2048, I=768,
E=128, top-8) decoding at batch 1 with k=136 (k/I ~ 17.8%), c=272, r=32,
tokens cycling through 20 seeded decode steps.  A step is one whole MoE-block
forward (route, rotate+quantize, screen, exact top-k, down+recovery,
combine).  Cache handling: the timed steps cycle through --layers distinct
device copies of the layer (32 by default, ~43 GB: inputs far larger than the
126 MB L2), so every step reads its weights from HBM, as a decode step through
a stack of layers does, while the kernel's code stays cached.  A second
measurement flushes the L2 between steps instead (a read of a 2x-L2 buffer,
outside the step events), which also evicts the kernel's code; it is reported
beside the headline as "l2_flush".  Timing: the steps run back to back in
chunks of 64, one event pair per chunk (a device spin ahead of each chunk lets
the host queue it whole), so consecutive launches overlap through programmatic
dependent launch as they do in a decode loop.

Metric: achieved HBM GB/s on the algorithmic bytes of the step (32-byte
sector accounting), plus us/step.  One JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-block µs/step & achieved HBM GB/s (vs ~8 TB/s) at k/I≈18%, batch 1–16"


def launches_per_step(B: int, path: int) -> int:
    """Kernel launches of one sparse step: the one-cluster reader routes inside
    its kernel at B <= 2 (one launch) and after the route and select kernels
    above (three); the streamed reader is route, select and five stage
    kernels."""
    streamed = path == 2 or (path == 0 and B > 2)
    if streamed:
        return 7
    return 1 if B <= 2 else 3


def workload_name(B: int) -> str:
    return f"qwen3_30b_a3b_layer_b{B}"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=4000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--batch", type=int, default=1)
    p.add_argument("--k", type=int, default=136)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--layers", type=int, default=32, help="distinct device copies of the layer the steps cycle through")
    p.add_argument("--path", type=int, default=0, choices=[0, 1, 2],
                   help="sparse reader: 0 automatic, 1 one cluster per expert, 2 streamed kernels")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("reader.cu", "common.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "calibration_free_channel_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    cur = kernel_source_hash()
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        f = dict(kv.split("=", 1) for kv in line.split())
        if f.get("kernel") == kernel and f.get("workload") == workload and f.get("source") == cur:
            return int(f["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return
        time.sleep(0.1)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                self.rows.append(f)

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ------------------------------------------------------------------ native
def run_native(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from calibration_free_channel_b200 import accounting, synth
    from calibration_free_channel_b200 import moe_reader as M

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    M.moe_reader_set_path(args.path)
    shape = synth.QWEN3_30B_A3B
    B, k, c, r = args.batch, args.k, 2 * args.k, 32
    W = synth.layer_weights(shape, seed=0, device=str(dev))
    layer = M.Layer(W, top_e=shape.top_e, device=dev).build_sketch(synth.rot_seed(0)).build_lowrank(r)
    # distinct device copies of the layer (same values, separate memory): the
    # timed steps cycle through them so the working set is far above the L2
    layers = [layer] + [replicate(layer) for _ in range(max(1, args.layers) - 1)]
    nlay = len(layers)
    ntok = 20
    toks = [synth.tokens(shape.d, B, seed=1000 * rank + s) for s in range(ntok)]
    xs = [t.to(dev) for t in toks]
    y = torch.empty_like(xs[0])

    # algorithmic bytes of each token's step (exact sector accounting of the
    # rows the reader reads, from its own debug outputs; untimed)
    step_bytes = []
    for x in xs:
        _, dbg = layer.forward(x, k=k, c=c, debug=True)
        ids, cand, kept = (dbg[n].cpu().numpy() for n in ("ids", "cand", "kept"))
        step_bytes.append(accounting.step_bytes(shape.E, shape.I, shape.d, r, ids, cand, kept)["total"])
    layer.check()
    expert_bytes = [b - accounting.router_bytes(shape.E, shape.d, False) for b in step_bytes]

    # L2 flush between timed steps: READ a buffer of twice the L2 size, so the
    # L2 holds only clean lines afterwards (a write-flush would leave ~L2-size
    # of dirty lines whose write-back then competes with the step's reads)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.ones(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    flush_out = torch.empty((), dtype=torch.float32, device=dev)

    class _Flush:
        @staticmethod
        def zero_():
            torch.sum(flush_buf, dim=0, out=flush_out)

    flush = _Flush()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    chunk = 64
    spin_cycles = int(2.0e9 * chunk * 150e-6)  # ~150 us of host time per step, at up to 2 GHz

    def time_loop(fn, steps, warmup, kernel_events=False, flushed=False):
        for i in range(warmup):
            if flushed:
                flush.zero_()
            fn(i)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)] \
            if kernel_events else None
        if kev:  # create the underlying CUDA events before handing them to the library
            for a_, b_ in kev:
                a_.record()
                b_.record()
        barrier()
        with ClockSampler(local_rank) as cs:
            for i in range(steps):
                if i % chunk == 0:
                    # a device-side spin ahead of each chunk of steps: the host
                    # queues the whole chunk before the GPU reaches it, so the
                    # per-step events time the device, not the Python launch path
                    torch.cuda._sleep(spin_cycles)
                if flushed:
                    flush.zero_()
                if kev:
                    M.moe_reader_set_expert_events(kev[i][0], kev[i][1])
                ev[i][0].record()
                fn(i)
                ev[i][1].record()
            barrier()
        M.moe_reader_set_expert_events(None, None)
        per = [a.elapsed_time(b) for a, b in ev]
        kper = [a.elapsed_time(b) for a, b in kev] if kev else None
        return per, kper, cs.summary()

    def chunk_loop(fn, steps, warmup):
        """Back-to-back steps timed per chunk of `chunk` steps (one event pair
        per chunk, a device spin ahead of it so the host has queued the whole
        chunk): nothing but the steps' own kernels runs between the events, so
        consecutive launches overlap as they do in a decode loop.  Returns the
        mean time per step of each chunk (ms)."""
        for i in range(warmup):
            fn(i)
        nch = max(1, steps // chunk)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nch)]
        barrier()
        with ClockSampler(local_rank) as cs:
            for q in range(nch):
                torch.cuda._sleep(spin_cycles)
                ev[q][0].record()
                for i in range(q * chunk, (q + 1) * chunk):
                    fn(i)
                ev[q][1].record()
            barrier()
        return [a.elapsed_time(b) / chunk for a, b in ev], nch * chunk, cs.summary()

    def sparse_step(j):
        layers[j % nlay].forward(xs[j % ntok], k=k, c=c, out=y)

    def sparse_step_one_layer(j):
        layer.forward(xs[j % ntok], k=k, c=c, out=y)

    per, nsteps, clocks = chunk_loop(sparse_step, args.steps, args.warmup)
    # the expert launch alone (events right around it inside the library): it
    # separates the kernel from the step, at the cost of the launch overlap
    _, kper, _ = time_loop(sparse_step, max(64, args.steps // 8), args.warmup, kernel_events=True)
    fper, fkper, _ = time_loop(sparse_step_one_layer, max(50, args.steps // 4), args.warmup, kernel_events=True,
                               flushed=True)
    ms = statistics.mean(per)
    kms = statistics.mean(kper)
    mean_bytes = statistics.mean(step_bytes[i % ntok] for i in range(nsteps))
    mean_ebytes = statistics.mean(expert_bytes[i % ntok] for i in range(nsteps))
    # max over ranks
    t = torch.tensor([ms, kms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max, kms_max = float(t[0]), float(t[1])
    value = world * mean_bytes / (ms_max * 1e-3) / 1e9

    # end to end through the host-buffer C-ABI call: H2D x, step, D2H y
    xh = [t.pin_memory() for t in toks]
    yh = torch.empty_like(xh[0]).pin_memory()
    xd = torch.empty_like(xs[0])
    yd = torch.empty_like(xs[0])
    ws = layer.workspace(B)
    sts = [lay.struct() for lay in layers]

    def e2e_step(j):
        M.moe_reader_forward_host(sts[j % nlay], B, k, c, xh[j % ntok], xd, yd, yh, ws, ws.numel())

    e2e_steps = max(50, args.steps // 4)
    eper, _, _ = time_loop(e2e_step, e2e_steps, args.warmup)
    ems = statistics.mean(eper)
    t = torch.tensor([ems], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_value = world * mean_bytes / (float(t[0]) * 1e-3) / 1e9

    dense = None
    if not args.no_dense:
        def dense_step(j):
            layers[j % nlay].forward_dense(xs[j % ntok], out=y)
        dper, _, _ = chunk_loop(dense_step, max(64, args.steps // 4), args.warmup)
        dms = statistics.mean(dper)
        dbytes = accounting.router_bytes(shape.E, shape.d, False) + \
            shape.top_e * B * accounting.dense_expert_bytes(shape.I, shape.d) if B == 1 else None
        dense = {"us_per_step": dms * 1e3, "speedup_of_sparse": dms / ms,
                 "achieved_gbs": (dbytes / (dms * 1e-3) / 1e9) if dbytes else None}
    # the exact-input recovery (dropped candidates enter V z with their exact
    # a): same bytes, the down stage walks every candidate
    variant = None
    if r > 0:
        def variant_step(j):
            layers[j % nlay].forward(xs[j % ntok], k=k, c=c, out=y, recovery_input=1)
        vper, _, _ = chunk_loop(variant_step, max(64, args.steps // 4), args.warmup)
        variant = {"us_per_step": statistics.mean(vper) * 1e3}
    layer.check()

    peak, peak_kind = measured_peaks()
    # At B <= 2 the expert kernel routes in-kernel: it is the step's only
    # kernel and reads the router too, so a launch's bytes are the step's and
    # its average duration in the back-to-back chunks is the step time.  At
    # larger B the route/select kernels run first; the expert kernel's share
    # is timed with events right around its launch.
    fused = B <= 2 and args.path != 2
    launch_bytes = mean_bytes if fused else mean_ebytes
    launch_ms = ms_max if fused else kms_max
    achieved = launch_bytes / (launch_ms * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": nsteps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "us_per_step": ms_max * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 (int8 x 2-bit sketch dots, fp32 accumulate)",
        "data": "synthetic (seeded; Qwen3-30B-A3B layer shape, lognormal channel scales, Student-t tokens)",
        "config": {"workload": workload_name(B), "d": shape.d, "I": shape.I, "E": shape.E, "top_e": shape.top_e,
                   "batch": B, "k": k, "c": c, "r": r, "decode_steps_cycled": ntok,
                   "l2": f"inputs larger than L2: steps cycle through {nlay} distinct device copies of the layer "
                         f"({nlay * layer_bytes(layer) / 1e9:.1f} GB)",
                   "parallelism": f"replicas x{world}", "algorithmic_bytes_per_step": mean_bytes},
        "roofline": {"bound": "hbm", "kernel": "reader_kernel" if fused else "streamed kernels (screen .. down)",
                     "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)",
                     "bytes_per_launch": launch_bytes, "launch_us": launch_ms * 1e3,
                     "isolated_launch_us": kms_max * 1e3,
                     "traffic": profiled_traffic("reader_kernel", workload_name(B)) if fused else None},
        "step_roofline_frac": round(value / world / peak, 4),
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": B * shape.d * 2,
                "d2h_bytes_per_step": B * shape.d * 2, "us_per_step": float(t[0]) * 1e3},
        "gpu_launches": launches_per_step(B, args.path) * nsteps,
        "clocks": clocks,
        "dense": dense,
        "recovery_exact_input": variant,
        "l2_flush": {"us_per_step": statistics.mean(fper) * 1e3, "kernel_us": statistics.mean(fkper) * 1e3,
                     "note": "one layer, L2 flushed before every step (also evicts the kernel code)"},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(W, toks[:4], k, c, r, shape, budget_s=15.0)
    return out


def replicate(layer):
    """A copy of a reader layer in separate device memory (same values)."""
    import copy
    L = copy.copy(layer)
    L.w = {n: (v.clone() if v is not None else None) for n, v in layer.w.items()}
    for n in ("rot_sign", "sk_gate", "sk_up", "alpha_gate", "alpha_up", "u_sigma", "v"):
        t = getattr(layer, n, None)
        setattr(L, n, t.clone() if t is not None else None)
    return L


def layer_bytes(layer) -> int:
    tot = sum(v.numel() * v.element_size() for v in layer.w.values() if v is not None)
    for n in ("rot_sign", "sk_gate", "sk_up", "alpha_gate", "alpha_up", "u_sigma", "v"):
        t = getattr(layer, n, None)
        if t is not None:
            tot += t.numel() * t.element_size()
    return tot


# -------------------------------------------------------------- CPU oracle
def _oracle_setup(W_host, shape, r, toks, rot_seed):
    from oracle import oracle as O
    sk = O.build_sketch(W_host["w_gate"], W_host["w_up"], rot_seed)
    experts = set()
    for x in toks:
        _, ids, _ = O.route(x, W_host["w_router"], W_host.get("router_bias"), shape.top_e)
        experts |= set(ids.ravel().tolist())
    lr = O.build_lowrank(W_host["w_down"], r, experts=sorted(experts))
    return sk, lr


def _oracle_time(W_host, sk, lr, toks, k, c, r, shape, budget_s):
    from calibration_free_channel_b200 import accounting
    from oracle import oracle as O
    n = 0
    nbytes = 0
    t0 = time.perf_counter()
    while True:
        x = toks[n % len(toks)]
        _, _, dbg = O.forward(x, W_host, sk, lr, k=k, c=c, r=r, top_e=shape.top_e, debug=True)
        nbytes += accounting.step_bytes(shape.E, shape.I, shape.d, r, dbg["ids"], dbg["cand"], dbg["kept"])["total"]
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 200:
            return n, nbytes, el


def cpu_baseline(W, toks, k, c, r, shape, budget_s):
    W_host = {n: (v.cpu() if v is not None else None) for n, v in W.items()}
    from calibration_free_channel_b200 import synth
    sk, lr = _oracle_setup(W_host, shape, r, toks, synth.rot_seed(0))
    n, nbytes, el = _oracle_time(W_host, sk, lr, toks, k, c, r, shape, budget_s)
    return {"value": round(nbytes / el / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "us_per_step": el / n * 1e6,
            "sample": f"{n} decode steps of the same layer and tokens, single-threaded plain C oracle "
                      f"(fp64 exact stage; sketch/SVD build excluded), {el:.1f} s"}


def run_reference(args, rank, world):
    """The oracle timed on the host cores, same workload and metric."""
    if rank != 0:
        return None
    from calibration_free_channel_b200 import synth
    shape = synth.QWEN3_30B_A3B
    B, k, c, r = args.batch, args.k, 2 * args.k, 32
    W = synth.layer_weights(shape, seed=0)
    toks = [synth.tokens(shape.d, B, seed=s) for s in range(4)]
    sk, lr = _oracle_setup(W, shape, r, toks, synth.rot_seed(0))
    # each step: one whole decode step of the oracle; the run stops after K
    # steps or a 120 s budget, whichever comes first (a bounded sample)
    for w in range(min(args.warmup, 2)):
        _oracle_time(W, sk, lr, toks[w % 4:w % 4 + 1], k, c, r, shape, 0.0)
    tot_n = tot_b = 0
    tot_t = 0.0
    while tot_n < args.steps and tot_t < 120.0:
        n, nb, el = _oracle_time(W, sk, lr, toks[tot_n % 4:tot_n % 4 + 1], k, c, r, shape, 0.0)
        tot_n, tot_b, tot_t = tot_n + n, tot_b + nb, tot_t + el
    value = tot_b / tot_t / 1e9
    cb = {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
          "sample": f"{tot_n} decode steps (of {args.steps} asked, 120 s cap), single-threaded plain C oracle, "
                    f"tokens 0-3; sketch/SVD build excluded"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / tot_n * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32 (oracle)",
            "data": "synthetic", "config": {"workload": workload_name(B), "batch": B, "k": k, "c": c, "r": r},
            "cpu_baseline": cb,
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    out = run_native(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
