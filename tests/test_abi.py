"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host before anything is enqueued (no GPU
needed for any of these)."""
import ctypes as C
import os
import re

import pytest

from calibration_free_channel_b200 import build as Bld
from calibration_free_channel_b200 import moe_reader as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_reader.h")


@pytest.fixture(scope="module")
def lib():
    Bld.build()
    return M.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_reader_\w+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(M.EXPORTS)


def declared_arity():
    """Parameter count of every moe_reader_* prototype in the header."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(moe_reader_\w+)\s*\(([^)]*)\)\s*;", src):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_prototypes(lib):
    arity = declared_arity()
    assert sorted(arity) == declared_functions()
    for name, n in arity.items():
        assert len(getattr(lib, name).argtypes or []) == n, name


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_workspace_sizes_are_positive(lib):
    assert M.moe_reader_workspace_bytes(1, 128, 8, 768, 2048, 136, 272, 32) > 0
    assert M.moe_reader_workspace_bytes(64, 128, 8, 768, 2048, 136, 272, 32) > \
        M.moe_reader_workspace_bytes(1, 128, 8, 768, 2048, 136, 272, 32)
    assert M.moe_reader_lowrank_workspace_bytes(128, 768, 2048, 32) >= 128 * 768 * 768 * 4


def _layer(**kw):
    fake = 0x10000  # 16-byte aligned, never dereferenced: validation runs first
    base = dict(E=8, I=128, d=256, top_e=2, r=8, w_router=fake, router_bias=None, w_gate=fake, w_up=fake,
                w_down=fake, rot_sign=fake, sk_gate=fake, sk_up=fake, alpha_gate=fake, alpha_up=fake,
                u_sigma=fake, v=fake)
    base.update(kw)
    return M.MoeReaderLayer(**base)


def _fwd(lib, layer, B=1, k=24, c=48, x=0x10000, y=0x10000, ws=0x10000, nb=1 << 30):
    return lib.moe_reader_forward(C.byref(layer), B, k, c, x, None, y, None, ws, nb, None)


@pytest.mark.parametrize("kw,args", [
    (dict(d=200), {}), (dict(d=64), {}), (dict(d=8192), {}),
    (dict(I=8), {}), (dict(top_e=9), {}), (dict(E=2000), {}),
    (dict(r=12), {}), (dict(r=136), {}),
    (dict(w_gate=None), {}), (dict(sk_up=None), {}), (dict(u_sigma=None), {}),
    (dict(w_down=0x10008), {}),
    ({}, dict(k=0)), ({}, dict(k=129, c=129)), ({}, dict(c=23)), ({}, dict(c=129)),
    ({}, dict(B=0)), ({}, dict(B=300)), ({}, dict(x=None)), ({}, dict(y=0x10004)),
    ({}, dict(ws=None)), ({}, dict(nb=16)),
])
def test_forward_rejects_bad_arguments(lib, kw, args):
    assert _fwd(lib, _layer(**kw), **args) == M.MOE_EINVAL
    assert lib.moe_reader_last_error()


@pytest.mark.parametrize("kw", [dict(path=3), dict(path=-1), dict(cluster_size=1), dict(cluster_size=17),
                                dict(recovery_input=2)])
def test_forward_rejects_bad_options(lib, kw):
    assert _fwd(lib, _layer(**kw)) == M.MOE_EINVAL
    assert lib.moe_reader_last_error()


def test_forward_rejects_bad_test_hook(lib):
    dbg = M.MoeReaderDebug()
    dbg.withhold_copy = 2
    st = lib.moe_reader_forward(C.byref(_layer()), 1, 24, 48, 0x10000, None, 0x10000, C.byref(dbg), 0x10000,
                                1 << 30, None)
    assert st == M.MOE_EINVAL and b"withhold_copy" in lib.moe_reader_last_error()


def test_one_cluster_reader_limits(lib):
    # the one-cluster reader runs one or two tokens with d <= 2048; asking for
    # it above that is refused before anything is enqueued
    assert _fwd(lib, _layer(path=1), B=3) == M.MOE_EUNSUPPORTED
    assert b"B <= 2" in lib.moe_reader_last_error()
    assert _fwd(lib, _layer(path=1, d=4096), B=1) == M.MOE_EUNSUPPORTED


def test_layer_struct_layout():
    # the binding's structs match the header's field order and sizes
    assert [n for n, _ in M.MoeReaderLayer._fields_][-5:] == ["recovery_input", "path", "cluster_size",
                                                             "sketch_format", "expert_slot"]
    assert C.sizeof(M.MoeReaderLayer) == 5 * 4 + 4 + 12 * C.sizeof(C.c_void_p) + 4 * 4 + C.sizeof(C.c_void_p)
    assert [n for n, _ in M.MoeReaderDebug._fields_][-4:] == ["ev_before", "ev_after", "wait_limit_us",
                                                            "withhold_copy"]
    assert C.sizeof(M.MoeReaderDebug) == 12 * C.sizeof(C.c_void_p) + 8


def test_forward_without_recovery_needs_no_factors(lib):
    # r = 0: the factor pointers may be NULL; validation passes up to the
    # workspace-size check, which fails here on purpose (nothing launches).
    st = _fwd(lib, _layer(r=0, u_sigma=None, v=None), nb=16)
    assert st == M.MOE_EINVAL and b"workspace" in lib.moe_reader_last_error()


def test_sketch_format_is_validated(lib):
    assert _fwd(lib, _layer(sketch_format=2)) == M.MOE_EINVAL
    assert b"sketch_format" in lib.moe_reader_last_error()


def test_sketch_row_bytes(lib):
    # 2-bit codes: d / 4; base 3: ceil(d / 5) rounded up to whole 32-byte sectors
    assert M.moe_reader_sketch_row_bytes(2048, 0) == 512
    assert M.moe_reader_sketch_row_bytes(2048, 1) == 416
    assert M.moe_reader_sketch_row_bytes(256, 1) == 64
    assert M.moe_reader_sketch_row_bytes(4096, 1) == 832
    assert M.moe_reader_sketch_row_bytes(2048, 2) == 0
    assert M.moe_reader_sketch_row_bytes(100, 1) == 0


def test_build_calls_validate(lib):
    f = 0x10000
    assert lib.moe_reader_build_sketch(8, 128, 100, f, f, 1, f, f, f, f, f, None) == M.MOE_EINVAL
    assert lib.moe_reader_build_sketch(8, 128, 256, None, f, 1, f, f, f, f, f, None) == M.MOE_EINVAL
    assert lib.moe_reader_build_lowrank(8, 128, 256, 12, f, f, f, f, 1 << 40, None) == M.MOE_EINVAL
    assert lib.moe_reader_build_lowrank(8, 128, 256, 96, f, f, f, f, 1 << 40, None) == M.MOE_EUNSUPPORTED
    assert lib.moe_reader_build_lowrank(8, 128, 256, 8, f, f, f, f, 16, None) == M.MOE_EINVAL
    assert lib.moe_reader_rmsnorm(1, 256, -1.0, f, f, None) == M.MOE_EINVAL
    assert lib.moe_reader_sketch_to_base3(8, 128, 100, f, f, None) == M.MOE_EINVAL
    assert lib.moe_reader_sketch_to_base3(8, 128, 256, None, f, None) == M.MOE_EINVAL
    assert lib.moe_reader_forward_dense(C.byref(_layer(w_up=None)), 1, f, None, f, f, 1 << 30, None) == M.MOE_EINVAL


def test_binding_raises_with_the_message(lib):
    with pytest.raises(M.MoeError, match="MOE_EINVAL.*d = 200"):
        M.moe_reader_forward(_layer(d=200), 1, 24, 48, 0x10000, None, 0x10000, None, 0x10000, 1 << 30)


def test_expert_slot_rules(lib):
    # the slot map is read by the streamed reader only: path 1 and the dense
    # block refuse it before anything is enqueued; it must be 16-byte aligned
    assert _fwd(lib, _layer(expert_slot=0x10000, path=1)) == M.MOE_EUNSUPPORTED
    assert b"expert_slot" in lib.moe_reader_last_error()
    st = lib.moe_reader_forward_dense(C.byref(_layer(expert_slot=0x10000)), 1, 0x10000, None, 0x10000, 0x10000,
                                      1 << 30, None)
    assert st == M.MOE_EUNSUPPORTED
    assert _fwd(lib, _layer(expert_slot=0x10004)) == M.MOE_EINVAL
