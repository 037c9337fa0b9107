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


def launches_per_step(B: int, path: int, d: int = 2048) -> int:
    """Kernel launches of one sparse step: the one-cluster reader (B <= 2,
    d <= 2048) routes inside its one kernel; the streamed reader is the route
    and select kernels and five stage kernels."""
    cluster = path == 1 or (path == 0 and B <= 2 and d <= 2048)
    return 1 if cluster else 7


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
    p.add_argument("--no-sweep", action="store_true", help="skip the batch and skewed-routing sweeps")
    p.add_argument("--layers", type=int, default=32, help="distinct device copies of the layer the steps cycle through")
    p.add_argument("--ep", action="store_true",
                   help="expert-parallel step: each rank holds only its experts e %% N == rank (compacted) and the "
                        "ranks sum their partials with one NCCL all-reduce of [B, d] fp32 per layer")
    p.add_argument("--sketch", default="2bit", choices=["2bit", "base3"],
                   help="sketch rows of the headline steps: 2-bit codes or base 3 (five trits per byte)")
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
    for name in ("reader.cu", "common.cuh", "kernels.h", "rotate.cuh", "select.cuh"):
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
    import torch
    import torch.distributed as dist

    from calibration_free_channel_b200 import accounting, synth
    from calibration_free_channel_b200 import moe_reader as M

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    shape = synth.QWEN3_30B_A3B
    B, k, c, r = args.batch, args.k, 2 * args.k, 32
    W = synth.layer_weights(shape, seed=0, device=str(dev))
    layer = M.Layer(W, top_e=shape.top_e, device=dev).build_sketch(synth.rot_seed(0)).build_lowrank(r)
    layer.path = args.path
    # distinct device copies of the layer (same values, separate memory): the
    # timed steps cycle through them so the working set is far above the L2
    layers = [layer] + [replicate(layer) for _ in range(max(1, args.layers) - 1)]
    nlay = len(layers)
    # every layer copy's workspace exists before any timing (sized for the
    # largest batch this run steps), so no allocation lands in a timed region
    for lay in layers:
        lay.workspace(max(B, 64))
    ntok = 20
    toks = [synth.tokens(shape.d, B, seed=1000 * rank + s) for s in range(ntok)]
    xs = [t.to(dev) for t in toks]
    y_bufs = {}

    def out_buf(Bq):
        if Bq not in y_bufs:
            y_bufs[Bq] = torch.empty((Bq, shape.d), dtype=torch.bfloat16, device=dev)
        return y_bufs[Bq]

    def step_accounting(lays, xq, kq, cq):
        """Algorithmic bytes of each token set's sparse step and of the dense
        block on the same routing (exact sector accounting of the rows the
        reader reads, from its own debug outputs; untimed)."""
        sb, db = [], []
        bias = lays[0].w.get("router_bias") is not None
        packing = "base3" if lays[0].sketch_format == 1 else "2bit"
        for x in xq:
            _, dbg = lays[0].forward(x, k=kq, c=cq, debug=True)
            ids, cand, kept = (dbg[n].cpu().numpy() for n in ("ids", "cand", "kept"))
            acc = accounting.step_bytes(shape.E, shape.I, shape.d, r, ids, cand, kept, bias=bias, packing=packing)
            sb.append(acc["total"])
            db.append(acc["dense"])
        lays[0].check()
        return sb, db

    def to_base3(lay):
        """A descriptor of the same layer whose sketch rows are base 3 (five
        trits per byte), repacked from its 2-bit codes in new device memory."""
        l3 = replicate_view(lay)
        rb = M.moe_reader_sketch_row_bytes(shape.d, 1)
        l3.sk_gate = torch.empty((shape.E, shape.I, rb), dtype=torch.uint8, device=dev)
        l3.sk_up = torch.empty_like(l3.sk_gate)
        M.moe_reader_sketch_to_base3(shape.E, shape.I, shape.d, lay.sk_gate, l3.sk_gate)
        M.moe_reader_sketch_to_base3(shape.E, shape.I, shape.d, lay.sk_up, l3.sk_up)
        l3.sketch_format = 1
        return l3

    if args.sketch == "base3":
        layers = [to_base3(lay) for lay in layers]
        layer = layers[0]

    step_bytes, dense_bytes = step_accounting(layers, xs, k, c)

    # L2 flush between timed steps: READ a buffer of twice the L2 size, so the
    # L2 holds only clean lines afterwards (a write-flush would leave ~L2-size
    # of dirty lines whose write-back then competes with the step's reads)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.ones(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    flush_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        torch.sum(flush_buf, dim=0, out=flush_out)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    chunk = 64
    spin_cycles = int(2.0e9 * chunk * 150e-6)  # ~150 us of host time per step, at up to 2 GHz

    def time_loop(fn, steps, warmup, kernel_events=False, flushed=False):
        """One event pair around every step (and, with kernel_events, one
        around the step's expert kernels inside the library)."""
        for i in range(warmup):
            if flushed:
                flush()
            fn(i, None)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)] \
            if kernel_events else None
        if kev:  # create the underlying CUDA events before handing them to the library
            for a_, b_ in kev:
                a_.record()
                b_.record()
        barrier()
        for i in range(steps):
            if i % chunk == 0:
                # a device-side spin ahead of each chunk of steps: the host
                # queues the whole chunk before the GPU reaches it, so the
                # per-step events time the device, not the Python launch path
                torch.cuda._sleep(spin_cycles)
            if flushed:
                flush()
            ev[i][0].record()
            fn(i, kev[i] if kev else None)
            ev[i][1].record()
        barrier()
        per = [a.elapsed_time(b) for a, b in ev]
        kper = [a.elapsed_time(b) for a, b in kev] if kev else None
        return per, kper

    def chunk_loop(fn, steps, warmup, sample_clocks=False):
        """Exactly `steps` back-to-back steps, timed per chunk of at most
        `chunk` steps (one event pair per chunk, a device spin ahead of it so
        the host has queued the whole chunk): nothing but the steps' own
        kernels runs between the events, so consecutive launches overlap as
        they do in a decode loop.  Returns the mean time per step (ms) and the
        clocks sampled during the timed region."""
        for i in range(warmup):
            fn(i)
        sizes = [chunk] * (steps // chunk) + ([steps % chunk] if steps % chunk else [])
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in sizes]
        barrier()
        cs = ClockSampler(local_rank) if sample_clocks else None
        if cs:
            cs.__enter__()
        i = 0
        for q, n in enumerate(sizes):
            torch.cuda._sleep(spin_cycles)
            ev[q][0].record()
            for _ in range(n):
                fn(i)
                i += 1
            ev[q][1].record()
        barrier()
        if cs:
            cs.__exit__(None, None, None)
        total = sum(a.elapsed_time(b) for a, b in ev)
        return total / steps, (cs.summary() if cs else None)

    def max_over_ranks(*vals):
        t = torch.tensor(vals, dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return [float(v) for v in t]

    # ---------------------------------------------------- the headline step
    def sparse_step(j, ev=None):
        layers[j % nlay].forward(xs[j % ntok], k=k, c=c, out=out_buf(B), events=ev)

    def sparse_step_one_layer(j, ev=None):
        layer.forward(xs[j % ntok], k=k, c=c, out=out_buf(B), events=ev)

    K = args.steps
    ms, clocks = chunk_loop(sparse_step, K, args.warmup, sample_clocks=True)
    # the expert kernels alone (events right around them inside the library):
    # they separate the kernels from the step, at the cost of the launch overlap
    _, kper = time_loop(sparse_step, max(64, K // 8), args.warmup, kernel_events=True)
    fper, fkper = time_loop(sparse_step_one_layer, max(64, K // 8), args.warmup, kernel_events=True, flushed=True)
    mean_bytes = statistics.mean(step_bytes[i % ntok] for i in range(K))
    ms_max, kms_max = max_over_ranks(ms, statistics.mean(kper))
    value = world * mean_bytes / (ms_max * 1e-3) / 1e9

    # end to end through the host-buffer C-ABI call: H2D x, step, D2H y
    xh = [t.pin_memory() for t in toks]
    yh = torch.empty_like(xh[0]).pin_memory()
    xd = torch.empty_like(xs[0])
    yd = torch.empty_like(xs[0])
    ws = layer.workspace(B)
    sts = [lay.struct() for lay in layers]

    def e2e_step(j, ev=None):
        M.moe_reader_forward_host(sts[j % nlay], B, k, c, xh[j % ntok], xd, yd, yh, ws, ws.numel())

    eper, _ = time_loop(e2e_step, max(64, K // 4), args.warmup)
    (ems,) = max_over_ranks(statistics.mean(eper))
    e2e_value = world * mean_bytes / (ems * 1e-3) / 1e9

    peak, peak_kind = measured_peaks()
    dense = None
    if not args.no_dense:
        def dense_step(j):
            layers[j % nlay].forward_dense(xs[j % ntok], out=out_buf(B))
        dms, _ = chunk_loop(dense_step, max(64, K), args.warmup)
        (dms,) = max_over_ranks(dms)
        dmean = statistics.mean(dense_bytes)
        dense = {"us_per_step": dms * 1e3, "speedup_of_sparse": dms / ms_max,
                 "achieved_gbs": dmean / (dms * 1e-3) / 1e9, "bytes_per_step": dmean,
                 "hbm_bound_us": dmean / (peak * 1e9) * 1e6,
                 "note": "this build's all-channel block on the same weights and routing"}
    # the exact-input recovery (dropped candidates enter V z with their exact
    # a): same bytes
    variant = None
    if r > 0:
        def variant_step(j):
            layers[j % nlay].forward(xs[j % ntok], k=k, c=c, out=out_buf(B), recovery_input=1)
        vms, _ = chunk_loop(variant_step, max(64, K), args.warmup)
        variant = {"us_per_step": vms * 1e3}
    layer.check()

    # ------------------------------------------------ batch sweeps (extra keys)
    def sweep(lays, batches, kq, seed0, with_dense=True):
        res = {}
        for Bq in batches:
            xq = [synth.tokens(shape.d, Bq, seed=seed0 + 100 * Bq + s).to(dev) for s in range(8)]
            sb, db = step_accounting(lays, xq, kq, 2 * kq)
            yq = out_buf(Bq)

            def sp(j, xq=xq, yq=yq):
                lays[j % len(lays)].forward(xq[j % len(xq)], k=kq, c=2 * kq, out=yq)

            sms, _ = chunk_loop(sp, 64, 4)
            (sms,) = max_over_ranks(sms)
            ent = {"sparse_us": sms * 1e3, "sparse_gbs": statistics.mean(sb) / (sms * 1e-3) / 1e9,
                   "sparse_bytes": statistics.mean(sb), "sparse_hbm_bound_us": statistics.mean(sb) / (peak * 1e9) * 1e6}
            if with_dense:
                def dn(j, xq=xq, yq=yq):
                    lays[j % len(lays)].forward_dense(xq[j % len(xq)], out=yq)
                dms_, _ = chunk_loop(dn, 64, 4)
                (dms_,) = max_over_ranks(dms_)
                ent.update(dense_us=dms_ * 1e3, dense_bytes=statistics.mean(db),
                           dense_hbm_bound_us=statistics.mean(db) / (peak * 1e9) * 1e6,
                           speedup_vs_dense=dms_ / sms)
            res[f"B{Bq}"] = ent
            lays[0].check()
        return res

    batch_sweep = skewed_sweep = None
    if not args.no_sweep:
        batch_sweep = {"k": k, "c": c, "note": "budget/batch sweep of the same layer (8 token sets per batch, "
                                                 "64 back-to-back steps, steps cycle through the layer copies)"}
        batch_sweep.update(sweep(layers, (4, 16), k, 5000 + 1000 * rank))
        if args.k == 136:
            batch_sweep["k100"] = sweep(layers, (1, 4, 8, 16), 100, 7000 + 1000 * rank, with_dense=False)
        # skewed routing prior: the same weights with a per-expert logit bias ~ N(0, 1)
        bias = synth.router_bias(shape, seed=1).to(dev)
        skewed = []
        for lay in layers:
            sl = replicate_view(lay)
            sl.w["router_bias"] = bias
            skewed.append(sl)
        skewed_sweep = {"k": k, "c": c, "note": "router logit bias ~ N(0,1) per expert; sparse vs this build's "
                                                  "dense block on the same weights"}
        skewed_sweep.update(sweep(skewed, (1, 8, 16, 32, 64), k, 9000 + 1000 * rank))

    # the same steps with base-3 sketch rows (five trits per byte) against the
    # 2-bit codes, on the same token sets and layer copies
    base3 = None
    if not args.no_sweep and args.sketch == "2bit":
        l3s = [to_base3(lay) for lay in layers]
        base3 = {"note": "sketch rows 1.6 bits per trit (base 3) against 2-bit codes; same weights, tokens and "
                         "layer copies, 64 back-to-back steps each"}
        for Bq in (1, 16):
            xq = [synth.tokens(shape.d, Bq, seed=11000 + 100 * Bq + s).to(dev) for s in range(8)]
            yq = out_buf(Bq)
            ent = {}
            for name, lays in (("2bit", layers), ("base3", l3s)):
                sb, _ = step_accounting(lays, xq, k, c)

                def sp(j, lays=lays, xq=xq, yq=yq):
                    lays[j % len(lays)].forward(xq[j % len(xq)], k=k, c=c, out=yq)

                tms, _ = chunk_loop(sp, 64, 4)
                (tms,) = max_over_ranks(tms)
                ent[name] = {"us_per_step": tms * 1e3, "bytes_per_step": statistics.mean(sb)}
            ent["sketch_bytes_per_expert"] = {
                "2bit": 2 * shape.I * accounting.sketch_row_bytes(shape.d, "2bit") + 8 * shape.I,
                "base3": 2 * shape.I * accounting.sketch_row_bytes(shape.d, "base3") + 8 * shape.I}
            base3[f"B{Bq}"] = ent
            l3s[0].check()
        del l3s

    fused = B <= 2 and args.path != 2
    # the one-cluster kernel of the step: the two-exchange kernel at one token
    # on 2-bit rows, the channel-owning kernel otherwise
    kname = "reader1_kernel" if B == 1 and args.sketch == "2bit" and args.path != 2 else "reader_kernel"
    # At B <= 2 the reader routes in-kernel: it is the step's only kernel and
    # reads the router too, so a launch's bytes are the step's and its average
    # duration in the back-to-back chunks is the step time.  Above, the
    # streamed kernels' share is timed with events right around them.
    launch_bytes = mean_bytes if fused else mean_bytes - accounting.router_bytes(shape.E, shape.d, False)
    launch_ms = ms_max if fused else kms_max
    achieved = launch_bytes / (launch_ms * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "us_per_step": ms_max * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 (int8 x %s sketch dots, fp32 accumulate)" % ("base-3" if args.sketch == "base3" else "2-bit"),
        "data": "synthetic (seeded; Qwen3-30B-A3B layer shape, lognormal channel scales, Student-t tokens)",
        "config": {"workload": workload_name(B), "d": shape.d, "I": shape.I, "E": shape.E, "top_e": shape.top_e,
                   "batch": B, "k": k, "c": c, "r": r, "decode_steps_cycled": ntok,
                   "l2": f"inputs larger than L2: steps cycle through {nlay} distinct device copies of the layer "
                         f"({nlay * layer_bytes(layer) / 1e9:.1f} GB)",
                   "parallelism": f"replicas x{world}", "algorithmic_bytes_per_step": mean_bytes,
                   "sketch": args.sketch},
        "roofline": {"bound": "hbm", "kernel": kname if fused else "streamed kernels (screen .. down)",
                     "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json), burst copy",
                     "bytes_per_launch": launch_bytes, "launch_us": launch_ms * 1e3,
                     "isolated_launch_us": kms_max * 1e3,
                     "traffic": profiled_traffic(kname, workload_name(B)) if fused else None},
        "step_roofline_frac": round(value / world / peak, 4),
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": B * shape.d * 2,
                "d2h_bytes_per_step": B * shape.d * 2, "us_per_step": ems * 1e3},
        "gpu_launches": launches_per_step(B, args.path) * K,
        "clocks": clocks,
        "dense": dense,
        "recovery_exact_input": variant,
        "l2_flush": {"us_per_step": statistics.mean(fper) * 1e3, "kernel_us": statistics.mean(fkper) * 1e3,
                     "note": "one layer, L2 flushed before every step (also evicts the kernel code)"},
        "batch_sweep": batch_sweep,
        "skewed_sweep": skewed_sweep,
        "base3_sketch": base3,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(W, toks[:4], k, c, r, shape, budget_s=12.0)
    return out


def run_ep(args, rank, world, local_rank):
    """Expert-parallel steps: every rank holds the router and only its own
    experts (e % world == rank, compacted with an expert_slot map), reads the
    pairs of those experts for the whole batch, and the partials meet in one
    NCCL all-reduce of [B, d] fp32; the finish adds nothing and rounds to bf16.
    Total work is fixed as N grows (strong scaling); each rank holds 1/N of
    the expert bytes."""
    import torch
    import torch.distributed as dist

    from calibration_free_channel_b200 import accounting, ep, synth
    from calibration_free_channel_b200 import moe_reader as M

    dev = torch.device("cuda", local_rank)
    shape = synth.QWEN3_30B_A3B
    B, k, c, r = args.batch, args.k, 2 * args.k, 32
    W = synth.layer_weights(shape, seed=0, device=str(dev))
    Wr, slot = ep.shard_weights(W, rank, world)
    del W
    layer = M.Layer(Wr, top_e=shape.top_e, device=dev, expert_slot=slot).build_sketch(synth.rot_seed(0))
    layer = layer.build_lowrank(r)
    layers = [layer] + [replicate(layer) for _ in range(max(1, args.layers) - 1)]
    nlay = len(layers)
    for lay in layers:  # no allocation inside the timed region
        lay.workspace(B)
    toks = [synth.tokens(shape.d, B, seed=s).to(dev) for s in range(20)]
    # bytes of the whole step (all ranks together): the full reader's sets,
    # from this rank's debug outputs of the owned pairs summed over the ranks
    sb = []
    for x in toks[:4]:
        _, dbg = layer.forward_ep(x, k, c, rank, world, debug=True)
        ids, cand, kept = (dbg[n].cpu().numpy() for n in ("ids", "cand", "kept"))
        own = (ids % world) == rank
        per = accounting.step_bytes(shape.E, shape.I, shape.d, r, ids, cand, kept)["per_expert"]
        mine = sum(v["total"] for e, v in per.items() if e % world == rank)
        t = torch.tensor([float(mine)], dtype=torch.float64, device=dev)
        dist.all_reduce(t)
        sb.append(float(t) + accounting.router_bytes(shape.E, shape.d, False))
        del own
    layer.check()
    held = sum(t.numel() * t.element_size() for t in (layer.w["w_gate"], layer.w["w_up"], layer.w["w_down"],
                                                     layer.sk_gate, layer.sk_up, layer.u_sigma, layer.v))

    def step(j):
        ep.ep_forward(layers[j % nlay], toks[j % 20], k, c)

    for j in range(args.warmup):
        step(j)
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for j in range(args.steps):
        step(j)
    e1.record()
    torch.cuda.synchronize()
    dist.barrier()
    ms = e0.elapsed_time(e1) / args.steps
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t)
    layer.check()
    mean_bytes = statistics.mean(sb)
    return {"metric": METRIC, "value": round(mean_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "us_per_step": ms * 1e3,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16 (int8 x 2-bit sketch dots, fp32 accumulate)",
            "data": "synthetic (seeded; Qwen3-30B-A3B layer shape, lognormal channel scales, Student-t tokens)",
            "config": {"workload": workload_name(B), "batch": B, "k": k, "c": c, "r": r,
                       "parallelism": f"ep{world}", "algorithmic_bytes_per_step": mean_bytes,
                       "expert_bytes_held_per_rank": held,
                       "l2": f"inputs larger than L2: steps cycle through {nlay} layer copies per rank"},
            "gpu_launches": (7 + 2) * args.steps,
            "note": "one all-reduce of [B, d] fp32 per step (NCCL), then the bf16 finish"}


def replicate_view(layer):
    """A second descriptor of the same device tensors (its own weight dict);
    it shares the layer's workspace (the two are stepped one after the other
    on one stream, never concurrently)."""
    import copy
    L = copy.copy(layer)
    L.w = dict(layer.w)
    return L


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


def _oracle_time(W_host, sk, lr, toks, k, c, r, shape, budget_s, threads=1, max_steps=200):
    from calibration_free_channel_b200 import accounting
    from oracle import oracle as O
    n = 0
    nbytes = 0
    t0 = time.perf_counter()
    while True:
        x = toks[n % len(toks)]
        _, _, dbg = O.forward(x, W_host, sk, lr, k=k, c=c, r=r, top_e=shape.top_e, debug=True, threads=threads)
        nbytes += accounting.step_bytes(shape.E, shape.I, shape.d, r, dbg["ids"], dbg["cand"], dbg["kept"],
                                        bias=W_host.get("router_bias") is not None)["total"]
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= max_steps:
            return n, nbytes, el


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(W, toks, k, c, r, shape, budget_s):
    """The oracle on the host cores: its OpenMP variant over (token, slot)
    pairs on every core (the reported value), and single-threaded."""
    W_host = {n: (v.cpu() if v is not None else None) for n, v in W.items()}
    from calibration_free_channel_b200 import synth
    sk, lr = _oracle_setup(W_host, shape, r, toks, synth.rot_seed(0))
    cores = host_cores()
    n, nbytes, el = _oracle_time(W_host, sk, lr, toks, k, c, r, shape, budget_s, threads=cores)
    n1, nb1, el1 = _oracle_time(W_host, sk, lr, toks, k, c, r, shape, budget_s / 2, threads=1)
    return {"value": round(nbytes / el / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "us_per_step": el / n * 1e6,
            "sample": f"{n} decode steps of the same layer and tokens, plain C oracle with its (token, slot) "
                      f"readers on {cores} OpenMP threads (fp64 exact stage; sketch/SVD build excluded), {el:.1f} s",
            "single_thread": {"value": round(nb1 / el1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "us_per_step": el1 / n1 * 1e6, "sample": f"{n1} decode steps, {el1:.1f} s"}}


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
    cores = host_cores()
    # each step: one whole decode step of the oracle on every core; the run
    # stops after K steps or a 120 s budget, whichever comes first (a bounded
    # sample)
    for w in range(min(args.warmup, 2)):
        _oracle_time(W, sk, lr, toks[w % 4:w % 4 + 1], k, c, r, shape, 0.0, threads=cores)
    tot_n = tot_b = 0
    tot_t = 0.0
    while tot_n < args.steps and tot_t < 120.0:
        n, nb, el = _oracle_time(W, sk, lr, toks[tot_n % 4:tot_n % 4 + 1], k, c, r, shape, 0.0, threads=cores)
        tot_n, tot_b, tot_t = tot_n + n, tot_b + nb, tot_t + el
    value = tot_b / tot_t / 1e9
    cb = {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
          "sample": f"{tot_n} decode steps (of {args.steps} asked, 120 s cap), plain C oracle on {cores} OpenMP "
                    f"threads, tokens 0-3; sketch/SVD build excluded"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": tot_n, "warmup": args.warmup, "ms_per_step": tot_t / tot_n * 1e3,
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
    if world > 1 or args.ep:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        if world == 1:  # a one-rank group for the expert-parallel exchange
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29531")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    out = run_ep(args, rank, world, local_rank) if args.ep else run_native(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1 or args.ep:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
