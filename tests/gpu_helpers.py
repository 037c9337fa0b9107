"""Shared helpers of the GPU parity tests: run the CUDA path through the
C ABI and the CPU oracle on the same seeded inputs, then compare.

The parity bar: routing ids, integer sketch dots, screening scores and
candidate sets bit-exact; kept sets equal except for swaps inside an oracle
boundary gap below 1e-3 relative; fp32 per-expert outputs within max-abs
2e-2; bf16 outputs within 2e-2 beyond half a bf16 ulp of the exact value and
rel-L2 1e-2 (fp32 accumulation, bf16 in and out)."""
from __future__ import annotations

import numpy as np
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from oracle import oracle as O

MAX_ABS, REL_L2, KEPT_GAP = 2e-2, 1e-2, 1e-3


class OracleCache:
    """Oracle-side sketch and low-rank factors of one layer (built from the
    weights by the oracle alone)."""

    def __init__(self, W, rot_seed, r):
        self.W = W
        self.sk = O.build_sketch(W["w_gate"], W["w_up"], rot_seed)
        self.r = r
        E, I, d = W["w_gate"].shape
        self.us = np.zeros((E, I, max(r, 1)), np.uint16)
        self.vv = np.zeros((E, d, max(r, 1)), np.uint16)
        self.built = set()
        self.wd = synth.bf16_bits(W["w_down"])

    def lowrank_for(self, experts):
        if self.r == 0:
            return None
        for e in sorted(set(int(e) for e in np.ravel(experts)) - self.built):
            ubar, V, _ = O.lowrank_f64(self.wd[e], self.r)
            self.us[e] = O.f64_to_bf16(ubar)
            self.vv[e] = O.f64_to_bf16(V)
            self.built.add(e)
        return self.us, self.vv


def exact_a(W, e, chans, xb):
    """The oracle's exact-stage a_i = silu_r(g_i) u_i for the given channels."""
    xf = O.bf16_to_f64(xb)
    g = (O.bf16_to_f64(W["w_gate"][e][chans]) @ xf).astype(np.float32)
    u = (O.bf16_to_f64(W["w_up"][e][chans]) @ xf).astype(np.float32)
    return np.array([np.float32(O.silu_r(float(gi))) * ui for gi, ui in zip(g, u)], np.float32)


def compare_step(W, x, gpu_y, gdbg, ora_y64, odbg, k, ora_logits=None, check_kept=True):
    """Asserts the parity bar; returns a dict of the measured errors."""
    B, top = odbg["ids"].shape
    g = {n: v.cpu().numpy() for n, v in gdbg.items()}
    ok_tok = []
    for b in range(B):
        if np.array_equal(g["ids"][b], odbg["ids"][b]):
            ok_tok.append(b)
            continue
        # a routing difference is accepted only at an fp64 near-tie of the logits
        L = ora_logits[b] if ora_logits is not None else None
        assert L is not None, f"token {b}: routing differs {g['ids'][b]} vs {odbg['ids'][b]}"
        srt = np.sort(L)[::-1]
        assert abs(srt[top - 1] - srt[top]) <= 1e-12 * abs(srt[top - 1]), f"token {b}: routing differs"
    assert len(ok_tok) >= B - 1
    tok = np.array(ok_tok)
    assert np.array_equal(g["dot_gate"][tok], odbg["dot_gate"][tok])
    assert np.array_equal(g["dot_up"][tok], odbg["dot_up"][tok])
    assert np.array_equal(g["score"][tok].view(np.uint32), odbg["score"][tok].view(np.uint32))
    assert np.array_equal(g["cand"][tok], odbg["cand"][tok])
    swaps = 0
    xb = synth.bf16_bits(x.cpu()) if isinstance(x, torch.Tensor) else x
    for b in tok:
        for s in range(top):
            G, Ok = set(g["kept"][b, s].tolist()), set(odbg["kept"][b, s].tolist())
            assert len(G) == k
            if G == Ok or not check_kept:
                continue
            cand = odbg["cand"][b, s]
            a = np.abs(exact_a(W, odbg["ids"][b, s], cand, xb[b]))
            srt = np.sort(a)[::-1]
            kth, k1 = srt[k - 1], srt[k]
            assert (kth - k1) <= KEPT_GAP * kth, f"kept sets differ outside a near-tie ({b},{s})"
            amap = dict(zip(cand.tolist(), a.tolist()))
            for i in G ^ Ok:
                assert k1 * (1 - 1e-6) <= amap[i] <= kth * (1 + 1e-6), f"channel {i} outside the tie band"
            swaps += 1
    # fp32 per-expert outputs (before the bf16 rounding) where the kept sets agree
    ye_err = 0.0
    if "y_expert" in odbg and odbg["y_expert"] is not None:
        for b in tok:
            for s in range(top):
                if set(g["kept"][b, s].tolist()) == set(odbg["kept"][b, s].tolist()):
                    d = np.abs(g["y_expert"][b, s].astype(np.float64) - odbg["y_expert"][b, s])
                    ye_err = max(ye_err, float(d.max()))
        assert ye_err <= MAX_ABS, f"fp32 expert output error {ye_err}"
    yg = gpu_y.float().cpu().numpy().astype(np.float64)[tok]
    yo = ora_y64[tok]
    diff = np.abs(yg - yo)
    err = float(diff.max())
    rel = float(np.linalg.norm(yg - yo) / max(np.linalg.norm(yo), 1e-30))
    # bf16 output: within 2e-2 beyond half a bf16 ulp of the exact value (half
    # an ulp is the error of rounding the exact value once to bf16)
    ulp = bf16_ulp(yo)
    excess = float((diff - 0.5 * ulp).max())
    assert excess <= MAX_ABS and rel <= REL_L2, dict(max_abs=err, excess=excess, rel=rel, ye_err=ye_err,
                                                     swaps=swaps, ymax=float(np.abs(yo).max()))
    return dict(max_abs=err, excess_over_ulp=excess, rel_l2=rel, y_expert_max_abs=ye_err, swaps=swaps)


def bf16_ulp(v):
    """One bf16 ulp at the magnitude of v (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def run_pair(layer: M.Layer, oc: OracleCache, x, k, c, top_e, use_oracle_factors=True, recovery_input=0):
    """One step on both sides.  With use_oracle_factors the GPU reads the
    oracle's low-rank factors (so both sides read identical inputs);
    otherwise it reads its own build."""
    W = oc.W
    logits, ids, _ = O.route(x, W["w_router"], W.get("router_bias"), top_e)
    lr = oc.lowrank_for(ids)
    if oc.r == 0:
        layer.set_lowrank(None, None)  # no recovery on either side
    elif use_oracle_factors:
        layer.set_lowrank(torch.from_numpy(lr[0].view(np.int16)).view(torch.bfloat16),
                          torch.from_numpy(lr[1].view(np.int16)).view(torch.bfloat16))
    y, dbg = layer.forward(x.cuda(), k=k, c=c, debug=True, recovery_input=recovery_input)
    layer.check()
    _, y64, odbg = O.forward(x, W, oc.sk, lr, k=k, c=c, r=oc.r, top_e=top_e, debug=True,
                             recovery_input=recovery_input)
    return y, dbg, y64, odbg, logits


def check_pair(layer, oc, x, k, c, top_e, use_oracle_factors=True, check_kept=True, recovery_input=0):
    y, dbg, y64, odbg, logits = run_pair(layer, oc, x, k, c, top_e, use_oracle_factors, recovery_input)
    return compare_step(oc.W, x, y, dbg, y64, odbg, k, ora_logits=logits, check_kept=check_kept)
