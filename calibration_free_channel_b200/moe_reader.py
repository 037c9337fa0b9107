"""Python binding of the C ABI in include/moe_reader.h.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch provides device memory and streams.  If the library is not
built, importing the functions raises; there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_reader.so")

MOE_OK, MOE_EINVAL, MOE_EUNSUPPORTED, MOE_ECUDA, MOE_ETIMEOUT, MOE_EDEVICE = range(6)
_STATUS = {0: "MOE_OK", 1: "MOE_EINVAL", 2: "MOE_EUNSUPPORTED", 3: "MOE_ECUDA", 4: "MOE_ETIMEOUT",
           5: "MOE_EDEVICE"}

EXPORTS = ["moe_reader_workspace_bytes", "moe_reader_build_sketch", "moe_reader_lowrank_workspace_bytes",
           "moe_reader_build_lowrank", "moe_reader_forward", "moe_reader_forward_dense",
           "moe_reader_forward_host", "moe_reader_rmsnorm", "moe_reader_check_error", "moe_reader_launch_plan",
           "moe_reader_forward_noalloc", "moe_reader_forward_ep", "moe_reader_ep_finish", "moe_reader_last_error",
           "moe_reader_sketch_row_bytes", "moe_reader_sketch_to_base3"]


class MoeReaderLayer(C.Structure):
    _fields_ = [("E", C.c_int32), ("I", C.c_int32), ("d", C.c_int32), ("top_e", C.c_int32), ("r", C.c_int32),
                ("w_router", C.c_void_p), ("router_bias", C.c_void_p), ("w_gate", C.c_void_p),
                ("w_up", C.c_void_p), ("w_down", C.c_void_p), ("rot_sign", C.c_void_p),
                ("sk_gate", C.c_void_p), ("sk_up", C.c_void_p), ("alpha_gate", C.c_void_p),
                ("alpha_up", C.c_void_p), ("u_sigma", C.c_void_p), ("v", C.c_void_p),
                ("recovery_input", C.c_int32), ("path", C.c_int32), ("cluster_size", C.c_int32),
                ("sketch_format", C.c_int32), ("expert_slot", C.c_void_p)]


class MoeReaderDebug(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("ids", "weights", "dot_gate", "dot_up", "score", "cand", "kept",
                                          "a_kept", "y_expert", "phase_ns", "ev_before", "ev_after")] + \
               [("wait_limit_us", C.c_uint32), ("withhold_copy", C.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with calibration_free_channel_b200.build.build()")
        L = C.CDLL(LIB_PATH)
        P, i32, sz = C.c_void_p, C.c_int, C.c_size_t
        L.moe_reader_workspace_bytes.restype = sz
        L.moe_reader_workspace_bytes.argtypes = [i32] * 8
        L.moe_reader_build_sketch.argtypes = [i32, i32, i32, P, P, C.c_uint64, P, P, P, P, P, P]
        L.moe_reader_lowrank_workspace_bytes.restype = sz
        L.moe_reader_lowrank_workspace_bytes.argtypes = [i32] * 4
        L.moe_reader_build_lowrank.argtypes = [i32, i32, i32, i32, P, P, P, P, sz, P]
        L.moe_reader_forward.argtypes = [C.POINTER(MoeReaderLayer), i32, i32, i32, P, P, P,
                                         C.POINTER(MoeReaderDebug), P, sz, P]
        L.moe_reader_forward_dense.argtypes = [C.POINTER(MoeReaderLayer), i32, P, P, P, P, sz, P]
        L.moe_reader_forward_ep.argtypes = [C.POINTER(MoeReaderLayer), i32, i32, i32, P, i32, i32, P,
                                            C.POINTER(MoeReaderDebug), P, sz, P]
        L.moe_reader_ep_finish.argtypes = [i32, i32, P, P, P, P]
        L.moe_reader_forward_host.argtypes = [C.POINTER(MoeReaderLayer), i32, i32, i32, P, P, P, P, P, sz, P]
        L.moe_reader_rmsnorm.argtypes = [i32, i32, C.c_float, P, P, P]
        L.moe_reader_check_error.argtypes = [P, P]
        L.moe_reader_launch_plan.argtypes = [i32] * 7 + [P]
        L.moe_reader_forward_noalloc.argtypes = [C.POINTER(MoeReaderLayer), i32, i32, i32, P, P, P, P]
        L.moe_reader_last_error.restype = C.c_char_p
        L.moe_reader_last_error.argtypes = []
        L.moe_reader_sketch_row_bytes.restype = sz
        L.moe_reader_sketch_row_bytes.argtypes = [i32, i32]
        L.moe_reader_sketch_to_base3.argtypes = [i32, i32, i32, P, P, P]
        for f in EXPORTS:
            if f not in ("moe_reader_workspace_bytes", "moe_reader_lowrank_workspace_bytes", "moe_reader_last_error",
                         "moe_reader_sketch_row_bytes"):
                getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != MOE_OK:
        raise MoeError(status, lib().moe_reader_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


# ------------------------------------------------------ the C ABI, by name
def moe_reader_workspace_bytes(B, E, top_e, I, d, k, c, r) -> int:
    return int(lib().moe_reader_workspace_bytes(B, E, top_e, I, d, k, c, r))


def moe_reader_lowrank_workspace_bytes(E, I, d, r) -> int:
    return int(lib().moe_reader_lowrank_workspace_bytes(E, I, d, r))


def moe_reader_build_sketch(E, I, d, w_gate, w_up, rot_seed, rot_sign, sk_gate, sk_up, alpha_gate, alpha_up,
                            stream=None):
    _check(lib().moe_reader_build_sketch(E, I, d, _ptr(w_gate), _ptr(w_up), rot_seed & ((1 << 64) - 1),
                                         _ptr(rot_sign), _ptr(sk_gate), _ptr(sk_up), _ptr(alpha_gate),
                                         _ptr(alpha_up), _stream(stream)))


def moe_reader_sketch_row_bytes(d, fmt) -> int:
    return int(lib().moe_reader_sketch_row_bytes(d, fmt))


def moe_reader_sketch_to_base3(E, I, d, sk_codes, sk_base3, stream=None):
    _check(lib().moe_reader_sketch_to_base3(E, I, d, _ptr(sk_codes), _ptr(sk_base3), _stream(stream)))


def moe_reader_build_lowrank(E, I, d, r, w_down, u_sigma, v, workspace, ws_bytes, stream=None):
    _check(lib().moe_reader_build_lowrank(E, I, d, r, _ptr(w_down), _ptr(u_sigma), _ptr(v), _ptr(workspace),
                                          ws_bytes, _stream(stream)))


def moe_reader_forward_ep(layer: MoeReaderLayer, B, k, c, x, ep_rank, ep_size, y_partial, dbg, workspace, ws_bytes,
                          stream=None):
    _check(lib().moe_reader_forward_ep(C.byref(layer), B, k, c, _ptr(x), ep_rank, ep_size, _ptr(y_partial),
                                       C.byref(dbg) if dbg is not None else None, _ptr(workspace), ws_bytes,
                                       _stream(stream)))


def moe_reader_ep_finish(B, d, y_sum, residual, y, stream=None):
    _check(lib().moe_reader_ep_finish(B, d, _ptr(y_sum), _ptr(residual), _ptr(y), _stream(stream)))


def moe_reader_forward(layer: MoeReaderLayer, B, k, c, x, residual, y, dbg, workspace, ws_bytes, stream=None):
    _check(lib().moe_reader_forward(C.byref(layer), B, k, c, _ptr(x), _ptr(residual), _ptr(y),
                                    C.byref(dbg) if dbg is not None else None, _ptr(workspace), ws_bytes,
                                    _stream(stream)))


def moe_reader_forward_dense(layer: MoeReaderLayer, B, x, residual, y, workspace, ws_bytes, stream=None):
    _check(lib().moe_reader_forward_dense(C.byref(layer), B, _ptr(x), _ptr(residual), _ptr(y), _ptr(workspace),
                                          ws_bytes, _stream(stream)))


def moe_reader_forward_noalloc(layer: MoeReaderLayer, B, k, c, x, residual, y, stream=None):
    """The step with the library's fixed device scratch (no workspace
    argument): for callers that cannot allocate device memory."""
    _check(lib().moe_reader_forward_noalloc(C.byref(layer), B, k, c, _ptr(x), _ptr(residual), _ptr(y),
                                            _stream(stream)))


def moe_reader_forward_host(layer: MoeReaderLayer, B, k, c, x_host, x_dev, y_dev, y_host, workspace, ws_bytes,
                            stream=None):
    _check(lib().moe_reader_forward_host(C.byref(layer), B, k, c, _ptr(x_host), _ptr(x_dev), _ptr(y_dev),
                                         _ptr(y_host), _ptr(workspace), ws_bytes, _stream(stream)))


def moe_reader_rmsnorm(B, d, eps, x, h, stream=None):
    _check(lib().moe_reader_rmsnorm(B, d, eps, _ptr(x), _ptr(h), _stream(stream)))


def moe_reader_check_error(workspace, stream=None):
    """workspace None: the error word of moe_reader_forward_noalloc's scratch."""
    _check(lib().moe_reader_check_error(_ptr(workspace), _stream(stream)))


def timing_debug(ev_before, ev_after) -> MoeReaderDebug:
    """A debug block that only records two torch.cuda.Event around the expert
    kernels of one call (no per-stage outputs)."""
    d = MoeReaderDebug()
    d.ev_before = ev_before.cuda_event
    d.ev_after = ev_after.cuda_event
    return d


def moe_reader_launch_plan(dense: bool, B, E, top_e, I, d, r) -> dict:
    out = (C.c_int32 * 4)()
    _check(lib().moe_reader_launch_plan(int(dense), B, E, top_e, I, d, r, C.cast(out, C.c_void_p)))
    return dict(cluster_size=out[0], ring_rows=out[1], smem_bytes=out[2], max_active_clusters=out[3])


# ----------------------------------------------------------- convenience
class Layer:
    """A resident MoE layer on the GPU: bf16 weights, the sketch and the
    low-rank map, with the C struct that describes them."""

    def __init__(self, weights: dict, top_e: int, device="cuda", expert_slot=None):
        """weights: w_router [E, d] (and router_bias [E]) for every expert;
        w_gate, w_up, w_down for all E experts, or (with expert_slot, [E]
        int32: the index of each expert in those arrays, -1 if not held) for
        the held experts only, compacted."""
        dev = torch.device(device)
        self.w = {k: (v.to(dev).contiguous() if v is not None else None) for k, v in weights.items()}
        Eh, I, d = self.w["w_gate"].shape
        E = self.w["w_router"].shape[0]
        if expert_slot is None and Eh != E:
            raise ValueError(f"{Eh} experts of weights for a router of {E}: pass expert_slot")
        self.E, self.E_held, self.I, self.d, self.top_e, self.r = E, Eh, I, d, top_e, 0
        self.rot_sign = torch.empty(d, dtype=torch.int8, device=dev)
        self.sk_gate = torch.empty((Eh, I, d // 16), dtype=torch.int32, device=dev)
        self.sk_up = torch.empty_like(self.sk_gate)
        self.alpha_gate = torch.empty((Eh, I), dtype=torch.float32, device=dev)
        self.alpha_up = torch.empty_like(self.alpha_gate)
        self.u_sigma = None
        self.v = None
        self._ws = None
        self.path = 0          # which reader runs a sparse step (see struct)
        self.sketch_format = 0  # 0: 2-bit codes, 1: base 3 (build_sketch(packing=...))
        # [E] int32 weight slot of each expert (held experts only, compacted), or None
        self.expert_slot = None if expert_slot is None else \
            torch.as_tensor(expert_slot, dtype=torch.int32).to(dev).contiguous()
        self.cluster_size = 0  # CTAs per cluster of the cluster kernels (0: automatic)

    def build_sketch(self, rot_seed: int, stream=None, packing: str = "2bit"):
        """packing "2bit": [E, I, d/16] words of 2-bit codes; "base3": [E, I,
        sketch_row_bytes] bytes, five trits per byte (the codes are built,
        repacked and dropped)."""
        if packing not in ("2bit", "base3"):
            raise ValueError(f"packing {packing!r}: use '2bit' or 'base3'")
        dev = self.w["w_gate"].device
        Eh = self.E_held
        if self.sk_gate.dtype != torch.int32:  # rebuilt after a base-3 packing
            self.sk_gate = torch.empty((Eh, self.I, self.d // 16), dtype=torch.int32, device=dev)
            self.sk_up = torch.empty_like(self.sk_gate)
        moe_reader_build_sketch(Eh, self.I, self.d, self.w["w_gate"], self.w["w_up"], rot_seed,
                                self.rot_sign, self.sk_gate, self.sk_up, self.alpha_gate, self.alpha_up, stream)
        self.sketch_format = 0
        if packing == "base3":
            rb = moe_reader_sketch_row_bytes(self.d, 1)
            g3 = torch.empty((Eh, self.I, rb), dtype=torch.uint8, device=dev)
            u3 = torch.empty_like(g3)
            moe_reader_sketch_to_base3(Eh, self.I, self.d, self.sk_gate, g3, stream)
            moe_reader_sketch_to_base3(Eh, self.I, self.d, self.sk_up, u3, stream)
            torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
            self.sk_gate, self.sk_up, self.sketch_format = g3, u3, 1
        return self

    def build_lowrank(self, r: int, stream=None):
        dev = self.w["w_down"].device
        Eh = self.E_held
        self.u_sigma = torch.empty((Eh, self.I, r), dtype=torch.bfloat16, device=dev)
        self.v = torch.empty((Eh, self.d, r), dtype=torch.bfloat16, device=dev)
        nb = moe_reader_lowrank_workspace_bytes(Eh, self.I, self.d, r)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        moe_reader_build_lowrank(Eh, self.I, self.d, r, self.w["w_down"], self.u_sigma, self.v, ws, nb, stream)
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
        del ws
        self.r = r
        return self

    def set_lowrank(self, u_sigma, v):
        """Use given factors ([E, I, r], [E, d, r] bf16) or none (None)."""
        if u_sigma is None:
            self.u_sigma = self.v = None
            self.r = 0
        else:
            dev = self.w["w_down"].device
            self.u_sigma = u_sigma.to(dev).contiguous()
            self.v = v.to(dev).contiguous()
            self.r = int(u_sigma.shape[-1])
        return self

    def struct(self, r: int | None = None, recovery_input: int = 0, path: int | None = None,
               cluster_size: int | None = None) -> MoeReaderLayer:
        """The C description of the layer.  path: 0 automatic, 1 one-cluster
        reader, 2 streamed reader (default: this layer's `path`);
        cluster_size: 0 automatic (default: this layer's `cluster_size`)."""
        rr = self.r if r is None else r
        return MoeReaderLayer(self.E, self.I, self.d, self.top_e, rr, _ptr(self.w["w_router"]),
                              _ptr(self.w.get("router_bias")), _ptr(self.w["w_gate"]), _ptr(self.w["w_up"]),
                              _ptr(self.w["w_down"]), _ptr(self.rot_sign), _ptr(self.sk_gate), _ptr(self.sk_up),
                              _ptr(self.alpha_gate), _ptr(self.alpha_up),
                              _ptr(self.u_sigma) if rr else None, _ptr(self.v) if rr else None, recovery_input,
                              self.path if path is None else path,
                              self.cluster_size if cluster_size is None else cluster_size, self.sketch_format,
                              _ptr(self.expert_slot))

    def shard(self, rank: int, world: int) -> "Layer":
        """What rank `rank` of a `world`-way expert-parallel step holds: the
        experts e % world == rank of this layer (weights, sketch, low-rank
        map) copied into new compacted arrays, the router whole, and
        expert_slot[e] = e // world for them, -1 elsewhere."""
        import copy
        dev = self.w["w_gate"].device
        own = torch.arange(rank, self.E, world, device=dev)
        S = copy.copy(self)
        S.w = {n: (v if v is None or n in ("w_router", "router_bias") else v.index_select(0, own).contiguous())
               for n, v in self.w.items()}
        for n in ("sk_gate", "sk_up", "alpha_gate", "alpha_up", "u_sigma", "v"):
            t = getattr(self, n)
            setattr(S, n, t.index_select(0, own).contiguous() if t is not None else None)
        slot = torch.full((self.E,), -1, dtype=torch.int32)
        slot[rank::world] = torch.arange(own.numel(), dtype=torch.int32)
        S.expert_slot = slot.to(dev)
        S.E_held = int(own.numel())
        S._ws = None
        return S

    def workspace(self, B: int):
        nb = moe_reader_workspace_bytes(B, self.E, self.top_e, self.I, self.d, 1, 1, self.r)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = torch.zeros(nb, dtype=torch.uint8, device=self.w["w_gate"].device)
        return self._ws

    def _debug(self, B, k, c, dev):
        P = (B, self.top_e)
        dbg_t = dict(ids=torch.empty(P, dtype=torch.int32, device=dev),
                     weights=torch.empty(P, dtype=torch.float32, device=dev),
                     dot_gate=torch.empty(P + (self.I,), dtype=torch.int32, device=dev),
                     dot_up=torch.empty(P + (self.I,), dtype=torch.int32, device=dev),
                     score=torch.empty(P + (self.I,), dtype=torch.float32, device=dev),
                     cand=torch.empty(P + (c,), dtype=torch.int32, device=dev),
                     kept=torch.empty(P + (k,), dtype=torch.int32, device=dev),
                     a_kept=torch.empty(P + (k,), dtype=torch.float32, device=dev),
                     y_expert=torch.empty(P + (self.d,), dtype=torch.float32, device=dev),
                     phase_ns=torch.zeros((B * self.top_e, 16), dtype=torch.int64, device=dev))
        dbg = MoeReaderDebug()
        for n, v in dbg_t.items():
            setattr(dbg, n, _ptr(v))
        return dbg_t, dbg

    def forward_ep(self, x, k: int, c: int, ep_rank: int, ep_size: int, debug: bool = False, r: int | None = None,
                   stream=None, out=None, recovery_input: int = 0):
        """This rank's fp32 partial of the block ([B, d]) over the experts
        e % ep_size == ep_rank; sum it over the ranks, then ep_finish."""
        B = x.shape[0]
        ws = self.workspace(B)
        yp = out if out is not None else torch.empty((B, self.d), dtype=torch.float32, device=x.device)
        dbg_t, dbg = self._debug(B, k, c, x.device) if debug else (None, None)
        moe_reader_forward_ep(self.struct(r, recovery_input), B, k, c, x, ep_rank, ep_size, yp, dbg, ws, ws.numel(),
                              stream)
        return (yp, dbg_t) if debug else yp

    def forward(self, x, k: int, c: int, residual=None, debug: bool = False, r: int | None = None, stream=None,
                out=None, recovery_input: int = 0, path: int | None = None, events=None):
        """events: (ev_before, ev_after) torch.cuda.Event recorded around the
        expert kernels (timing only; not with debug)."""
        B = x.shape[0]
        ws = self.workspace(B)
        y = out if out is not None else torch.empty_like(x)
        dbg_t, dbg = self._debug(B, k, c, x.device) if debug else (None, None)
        if events is not None:
            dbg = timing_debug(*events)
        moe_reader_forward(self.struct(r, recovery_input, path), B, k, c, x, residual, y, dbg, ws, ws.numel(),
                           stream)
        return (y, dbg_t) if debug else y

    def forward_dense(self, x, residual=None, stream=None, out=None):
        B = x.shape[0]
        ws = self.workspace(B)
        y = out if out is not None else torch.empty_like(x)
        moe_reader_forward_dense(self.struct(0), B, x, residual, y, ws, ws.numel(), stream)
        return y

    def check(self, stream=None):
        if self._ws is not None:
            moe_reader_check_error(self._ws, stream)
