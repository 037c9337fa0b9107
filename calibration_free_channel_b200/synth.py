"""Seeded synthetic inputs for the MoE block (weights, router, tokens).

This module only draws random numbers; it holds none of the reader's
arithmetic.  Both the CUDA path and the CPU oracle take their inputs from it.

The recipe stands in for the pages' models and benchmarks, which are not
available ("KAIST: MoE Decoding Needs No Calibration Data", section "Numbers
and limits", names Qwen3-30B-A3B-Thinking-2507 and others): only the
Qwen3-30B-A3B layer shape is used.

* gate, up, down weights ~ N(0, std = 1/sqrt(d)); every channel row of each
  matrix is scaled by its own lognormal(0, 1) draw;
* router weights ~ N(0, std = 1/sqrt(d)); optional logit bias ~ N(0, 1) per
  expert (a skewed routing prior);
* tokens x = RMSNorm(t) with t_j ~ Student-t(nu = 4), no gain, eps = 1e-6,
  computed in fp64 and rounded to bf16.

Every tensor is keyed by (seed, layer, tensor id, expert) through a Philox
counter-based generator (numpy), so any expert of any layer can be
regenerated alone.  `device="cuda"` draws with torch's device generator
instead (different values, same distributions) for large stacks.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass

import numpy as np
import torch

T_ROUTER, T_GATE, T_UP, T_DOWN, T_BIAS, T_TOKENS = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class BlockShape:
    E: int
    I: int
    d: int
    top_e: int


QWEN3_30B_A3B = BlockShape(E=128, I=768, d=2048, top_e=8)
TINY = BlockShape(E=8, I=128, d=256, top_e=2)


def _gen(seed: int, layer: int, tensor: int, expert: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, layer, tensor, expert])))


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _expert_matrix(seed: int, layer: int, tensor: int, e: int, I: int, d: int) -> torch.Tensor:
    g = _gen(seed, layer, tensor, e)
    w = g.standard_normal((I, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    scale = g.lognormal(0.0, 1.0, size=(I, 1)).astype(np.float32)
    return _to_bf16(w * scale)


def layer_weights(shape: BlockShape, seed: int = 0, layer: int = 0, bias: bool = False,
                  device: str = "cpu") -> dict:
    """Weights of one MoE layer: bf16 w_router [E,d], w_gate/w_up/w_down [E,I,d]
    (down stored channel-major, row i = channel i), fp32 router_bias [E] or None."""
    E, I, d = shape.E, shape.I, shape.d
    if device != "cpu":
        return _layer_weights_device(shape, seed, layer, bias, device)
    out = {}
    g = _gen(seed, layer, T_ROUTER, 0)
    out["w_router"] = _to_bf16(g.standard_normal((E, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d)))
    out["router_bias"] = (torch.from_numpy(_gen(seed, layer, T_BIAS, 0).standard_normal(E).astype(np.float32))
                          if bias else None)
    workers = min(16, os.cpu_count() or 1)
    for name, tid in (("w_gate", T_GATE), ("w_up", T_UP), ("w_down", T_DOWN)):
        t = torch.empty((E, I, d), dtype=torch.bfloat16)
        with _cf.ThreadPoolExecutor(workers) as ex:
            for e, m in enumerate(ex.map(lambda e: _expert_matrix(seed, layer, tid, e, I, d), range(E))):
                t[e] = m
        out[name] = t
    return out


def _layer_weights_device(shape: BlockShape, seed: int, layer: int, bias: bool, device: str) -> dict:
    E, I, d = shape.E, shape.I, shape.d
    g = torch.Generator(device=device)

    def key(tensor):
        return (seed * 1_000_003 + layer) * 16 + tensor

    out = {}
    g.manual_seed(key(T_ROUTER))
    out["w_router"] = (torch.randn((E, d), generator=g, device=device) / np.sqrt(d)).to(torch.bfloat16)
    if bias:
        g.manual_seed(key(T_BIAS))
        out["router_bias"] = torch.randn((E,), generator=g, device=device)
    else:
        out["router_bias"] = None
    for name, tid in (("w_gate", T_GATE), ("w_up", T_UP), ("w_down", T_DOWN)):
        g.manual_seed(key(tid))
        t = torch.empty((E, I, d), dtype=torch.bfloat16, device=device)
        for e in range(E):
            w = torch.randn((I, d), generator=g, device=device) / np.sqrt(d)
            s = torch.exp(torch.randn((I, 1), generator=g, device=device))
            t[e] = (w * s).to(torch.bfloat16)
        out[name] = t
    return out


def router_bias(shape: BlockShape, seed: int = 0, layer: int = 0) -> torch.Tensor:
    """The skewed routing prior alone: fp32 [E] ~ N(0, 1), the same values as
    layer_weights(..., bias=True) on the CPU draws for this seed and layer."""
    return torch.from_numpy(_gen(seed, layer, T_BIAS, 0).standard_normal(shape.E).astype(np.float32))


def tokens(d: int, B: int, seed: int = 0, layer: int = 0, dof: float | None = 4.0) -> torch.Tensor:
    """B tokens x = RMSNorm(t), t_j ~ Student-t(dof) (standard normal for
    dof=None), bf16 [B, d]."""
    g = _gen(seed, layer, T_TOKENS, 0)
    t = g.standard_t(dof, size=(B, d)) if dof is not None else g.standard_normal(size=(B, d))
    t = t / np.sqrt(np.mean(t * t, axis=1, keepdims=True) + 1e-6)
    return _to_bf16(t)


def rot_seed(seed: int = 0, layer: int = 0) -> int:
    """The rotation seed of a layer's sketch (a 64-bit integer)."""
    return int(np.random.SeedSequence([seed, layer, 99]).generate_state(1, dtype=np.uint64)[0])


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 view of a CPU bf16 tensor (what the oracle reads)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# The workloads (sizes and budgets); names say what they are.
WORKLOADS = {
    "tiny": dict(shape=TINY, B=1, k=24, c=48, r=8, seed=0),
    "qwen3_30b_a3b_layer_b1": dict(shape=QWEN3_30B_A3B, B=1, k=136, c=272, r=32, seed=0, steps=20),
    "qwen3_30b_a3b_budget_sweep": dict(shape=QWEN3_30B_A3B, B=(1, 4, 8, 16), k=(100, 136), r=32, seed=0),
    "qwen3_30b_a3b_batch_sweep_skewed": dict(shape=QWEN3_30B_A3B, B=(1, 8, 16, 32, 64), k=136, c=272, r=32,
                                             seed=0, bias=True),
    "qwen3_30b_a3b_stack48": dict(shape=QWEN3_30B_A3B, layers=48, B=(1, 16), k=136, c=272, r=32, seed=0),
}
