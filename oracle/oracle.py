"""Python face of the CPU oracle (TEST INFRASTRUCTURE ONLY).

Only tests, the smoke check and the bench's CPU-baseline / reference legs may
import this module.  It wraps the plain C oracle (moe_oracle.c) with ctypes
and adds the low-rank map, computed with numpy's LAPACK SVD in fp64.  It
shares no code with the CUDA library.

Page citations: "Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data", abstract (the reader: ternary-sketch screen, exact top-k,
low-rank recovery); "KAIST: MoE Decoding Needs No Calibration Data", section
"A reader that needs no data at all" (rotated ternary sketch of gate/up,
exact top-k from native BF16, low-rank map of the down projections).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
SRC_PATH = os.path.join(HERE, "moe_oracle.c")


def build(force: bool = False) -> str:
    """Compile the C oracle with strict IEEE semantics (no contraction)."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC_PATH):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11", "-fopenmp",
                               "-Wall", "-fPIC", "-shared", "-o", LIB_PATH, SRC_PATH, "-lm"])
    return LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB_PATH)
        P = C.c_void_p
        i32, u64, f32, f64 = C.c_int, C.c_uint64, C.c_float, C.c_double
        L.orc_splitmix64_at.restype = u64
        L.orc_splitmix64_at.argtypes = [u64, u64]
        L.orc_rot_signs.argtypes = [i32, u64, P]
        L.orc_fwht.argtypes = [i32, P]
        L.orc_exp_r.restype = f32
        L.orc_exp_r.argtypes = [f32]
        L.orc_silu_r.restype = f32
        L.orc_silu_r.argtypes = [f32]
        L.orc_double_to_bf16.restype = C.c_uint16
        L.orc_double_to_bf16.argtypes = [f64]
        L.orc_double_to_bf16_array.argtypes = [C.c_long, P, P]
        L.orc_rotate_quantize.argtypes = [i32, P, P, P, P, P]
        L.orc_twn_row.argtypes = [i32, P, P, P, P, P]
        L.orc_pack_trits.argtypes = [i32, P, P]
        L.orc_pack_trits_base3.argtypes = [i32, P, P]
        L.orc_unpack_trits_base3.argtypes = [i32, P, P]
        L.orc_unpack_trit.restype = i32
        L.orc_unpack_trit.argtypes = [P, i32]
        L.orc_build_sketch.argtypes = [i32, i32, i32, P, P, u64, P, P, P, P, P]
        L.orc_route.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P]
        L.orc_top_n.argtypes = [i32, P, P, i32, P]
        L.orc_expert_reader.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, f32, P, P, P, P,
                                        P, P, P, P, P, P, P, P, P, P, P, P]
        L.orc_forward.argtypes = [i32] * 10 + [P] * 25 + [i32]
        L.orc_forward_dense.argtypes = [i32] * 5 + [P] * 9
        L.orc_rmsnorm.argtypes = [i32, i32, f64, P, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _u16(a):
    """uint16 bf16 bits from a numpy uint16 array or a CPU bf16 torch tensor."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch
    return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(a) -> np.ndarray:
    a = _u16(a)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(a: np.ndarray) -> np.ndarray:
    flat = np.ascontiguousarray(np.asarray(a, dtype=np.float64).ravel())
    out = np.empty(flat.size, np.uint16)
    lib().orc_double_to_bf16_array(flat.size, _p(flat), _p(out))
    return out.reshape(np.shape(a))


# ------------------------------------------------------------- primitives
def splitmix64_at(seed: int, j: int) -> int:
    return int(lib().orc_splitmix64_at(seed, j))


def rot_signs(d: int, seed: int) -> np.ndarray:
    s = np.empty(d, np.int8)
    lib().orc_rot_signs(d, seed, _p(s))
    return s


def fwht(v: np.ndarray) -> np.ndarray:
    out = np.ascontiguousarray(v, dtype=np.float32).copy()
    lib().orc_fwht(out.size, _p(out))
    return out


def exp_r(t: float) -> float:
    return float(lib().orc_exp_r(float(t)))


def silu_r(t: float) -> float:
    return float(lib().orc_silu_r(float(t)))


def rotate_quantize(x, s: np.ndarray):
    x = _u16(x)
    d = x.size
    v = np.empty(d, np.float32)
    q = np.empty(d, np.int8)
    cx = np.zeros(1, np.float32)
    lib().orc_rotate_quantize(d, _p(x), _p(s), _p(v), _p(q), _p(cx))
    return v, q, float(cx[0])


def twn_row(w, s: np.ndarray):
    w = _u16(w)
    d = w.size
    t = np.empty(d, np.int8)
    a = np.zeros(1, np.float32)
    wrot = np.empty(d, np.float32)
    lib().orc_twn_row(d, _p(w), _p(s), _p(t), _p(a), _p(wrot))
    return t, float(a[0]), wrot


def pack_trits(trits: np.ndarray) -> np.ndarray:
    trits = np.ascontiguousarray(trits, np.int8)
    out = np.empty(trits.size // 16, np.uint32)
    lib().orc_pack_trits(trits.size, _p(trits), _p(out))
    return out


def pack_trits_base3(trits: np.ndarray) -> np.ndarray:
    """Five trits per byte (ceil(d / 5) bytes per row)."""
    trits = np.ascontiguousarray(trits, np.int8)
    out = np.empty((trits.size + 4) // 5, np.uint8)
    lib().orc_pack_trits_base3(trits.size, _p(trits), _p(out))
    return out


def unpack_trits_base3(packed: np.ndarray, d: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    out = np.empty(d, np.int8)
    lib().orc_unpack_trits_base3(d, _p(packed), _p(out))
    return out


def build_sketch(w_gate, w_up, rot_seed: int):
    """Sketch of every gate/up row: (rot_sign [d], sk_gate [E,I,d/16], sk_up,
    alpha_gate [E,I], alpha_up)."""
    wg, wu = _u16(w_gate), _u16(w_up)
    E, I, d = wg.shape
    s = np.empty(d, np.int8)
    skg = np.empty((E, I, d // 16), np.uint32)
    sku = np.empty_like(skg)
    ag = np.empty((E, I), np.float32)
    au = np.empty_like(ag)
    lib().orc_build_sketch(E, I, d, _p(wg), _p(wu), rot_seed, _p(s), _p(skg), _p(sku), _p(ag), _p(au))
    return s, skg, sku, ag, au


def route(x, w_router, bias=None, top_e: int = 8):
    x, wr = _u16(x), _u16(w_router)
    B, d = x.shape
    E = wr.shape[0]
    bias = None if bias is None else np.ascontiguousarray(np.asarray(bias, np.float32))
    logits = np.empty((B, E), np.float64)
    ids = np.empty((B, top_e), np.int32)
    w = np.empty((B, top_e), np.float32)
    lib().orc_route(B, E, d, top_e, _p(x), _p(wr), _p(bias), _p(logits), _p(ids), _p(w))
    return logits, ids, w


def top_n(keys: np.ndarray, n: int, idx: np.ndarray | None = None) -> np.ndarray:
    keys = np.ascontiguousarray(keys, np.float32)
    idx = np.arange(keys.size, dtype=np.int32) if idx is None else np.ascontiguousarray(idx, np.int32)
    out = np.empty(n, np.int32)
    lib().orc_top_n(idx.size, _p(idx), _p(keys), n, _p(out))
    return out


# --------------------------------------------------------------- low-rank map
def lowrank_f64(w_down_e, r: int):
    """Rank-r truncated SVD of one expert's W_down [I, d] in fp64:
    W = U S V^T, Ubar = U[:, :r] diag(S[:r]) [I, r], V = V[:, :r] [d, r].
    Sign rule: in each column the entry of V with the largest magnitude is
    positive (ties: lower index); Ubar's column flips with it.
    Reading: the pages name "a low-rank map of the down projections"; the
    rank-r SVD of W_down is the plainest such map."""
    W = bf16_to_f64(w_down_e) if not (isinstance(w_down_e, np.ndarray) and w_down_e.dtype == np.float64) \
        else w_down_e
    U, S, Vt = np.linalg.svd(W, full_matrices=False)
    ubar = U[:, :r] * S[:r]
    V = Vt[:r].T.copy()
    for p in range(r):
        j = int(np.argmax(np.abs(V[:, p])))
        if V[j, p] < 0:
            V[:, p] = -V[:, p]
            ubar[:, p] = -ubar[:, p]
    return ubar, V, S


def build_lowrank(w_down, r: int, experts=None):
    """bf16 factors for every expert (or only `experts`): u_sigma [E,I,r],
    v [E,d,r] as uint16 bf16 bits (zeros for experts not built)."""
    wd = _u16(w_down)
    E, I, d = wd.shape
    us = np.zeros((E, I, r), np.uint16)
    vv = np.zeros((E, d, r), np.uint16)
    for e in (range(E) if experts is None else experts):
        ubar, V, _ = lowrank_f64(wd[e], r)
        us[e] = f64_to_bf16(ubar)
        vv[e] = f64_to_bf16(V)
    return us, vv


# ---------------------------------------------------------------- forward
def forward(x, W: dict, sketch, lowrank, k: int, c: int, r: int, top_e: int,
            exact_mode: bool = False, residual=None, debug: bool = False, recovery_input: int = 0,
            threads: int = 1):
    """The sparse reader over B tokens.  Returns y (uint16 bf16 [B,d]), the
    fp64 output before rounding and (if debug) the per-stage values.
    recovery_input 1 feeds the low-rank map the exact a of dropped candidates
    (sketch estimates outside the candidate set); 0 sketch estimates for every
    skipped channel."""
    x = _u16(x)
    B, d = x.shape
    wr, wg, wu, wd = (_u16(W[n]) for n in ("w_router", "w_gate", "w_up", "w_down"))
    E, I, _ = wg.shape
    bias = W.get("router_bias")
    bias = None if bias is None else np.ascontiguousarray(np.asarray(bias, np.float32))
    s, skg, sku, ag, au = sketch
    us, vv = (None, None) if lowrank is None or r == 0 else (np.ascontiguousarray(lowrank[0]),
                                                             np.ascontiguousarray(lowrank[1]))
    res = None if residual is None else _u16(residual)
    y = np.empty((B, d), np.uint16)
    y64 = np.empty((B, d), np.float64)
    P = B * top_e
    dbg = dict(ids=np.empty((B, top_e), np.int32), weights=np.empty((B, top_e), np.float32),
               dot_gate=np.empty((B, top_e, I), np.int32), dot_up=np.empty((B, top_e, I), np.int32),
               score=np.empty((B, top_e, I), np.float32), cand=np.empty((B, top_e, c), np.int32),
               kept=np.empty((B, top_e, k), np.int32), a_kept=np.empty((B, top_e, k), np.float32),
               y_expert=np.empty((B, top_e, d), np.float64)) if debug else None
    g = (lambda n: _p(dbg[n])) if debug else (lambda n: None)
    assert P >= 1
    lib().orc_forward(B, E, top_e, I, d, k, c, r if us is not None else 0, int(exact_mode), int(recovery_input),
                      _p(x), _p(wr), _p(bias), _p(wg), _p(wu), _p(wd), _p(s), _p(skg), _p(sku),
                      _p(ag), _p(au), _p(us), _p(vv), _p(res), _p(y), _p(y64),
                      g("ids"), g("weights"), g("dot_gate"), g("dot_up"), g("score"), g("cand"),
                      g("kept"), g("a_kept"), g("y_expert"), int(threads))
    return y, y64, dbg


def forward_dense(x, W: dict, top_e: int, residual=None):
    x = _u16(x)
    B, d = x.shape
    wr, wg, wu, wd = (_u16(W[n]) for n in ("w_router", "w_gate", "w_up", "w_down"))
    E, I, _ = wg.shape
    bias = W.get("router_bias")
    bias = None if bias is None else np.ascontiguousarray(np.asarray(bias, np.float32))
    res = None if residual is None else _u16(residual)
    y = np.empty((B, d), np.uint16)
    y64 = np.empty((B, d), np.float64)
    lib().orc_forward_dense(B, E, top_e, I, d, _p(x), _p(wr), _p(bias), _p(wg), _p(wu), _p(wd),
                            _p(res), _p(y), _p(y64))
    return y, y64


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    x = _u16(x)
    B, d = x.shape
    h = np.empty_like(x)
    lib().orc_rmsnorm(B, d, eps, _p(x), _p(h))
    return h
