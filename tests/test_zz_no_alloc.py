"""moe_reader_forward_noalloc: the step with the library's fixed device
scratch instead of a caller-allocated workspace, for callers that cannot
allocate device memory (serving loops that forbid any allocation after
start-up so their footprint stays fixed, hosts whose device memory belongs to
another runtime's allocator).  Its outputs must match moe_reader_forward's on
the same inputs, on two calls in a row (the scratch persists between calls),
and the scratch's device error word must read clear afterwards.

This file is collected last on purpose, so a stop-at-first-failure run has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from tests.gpu_helpers import MAX_ABS, REL_L2, bf16_ulp

pytestmark = pytest.mark.gpu


def _close(y, ref):
    # both outputs are bf16 roundings of fp32 sums in different orders: they
    # may sit one bf16 ulp apart at a rounding boundary
    yg = y.float().cpu().numpy().astype(np.float64)
    yr = ref.float().cpu().numpy().astype(np.float64)
    assert (np.abs(yg - yr) - bf16_ulp(yr)).max() <= MAX_ABS
    assert np.linalg.norm(yg - yr) <= REL_L2 * np.linalg.norm(yr)


@pytest.mark.parametrize("B", [1, 4])
def test_noalloc_matches_forward_twice(B):
    W = synth.layer_weights(synth.TINY, seed=0)
    layer = M.Layer(W, top_e=2).build_sketch(synth.rot_seed(0)).build_lowrank(8)
    x = synth.tokens(256, B, seed=31).cuda()
    ref = layer.forward(x, k=24, c=48)
    st = layer.struct()
    for _ in range(2):
        y = torch.empty_like(x)
        M.moe_reader_forward_noalloc(st, B, 24, 48, x, None, y)
        torch.cuda.synchronize()
        _close(y, ref)
    M.moe_reader_check_error(None)  # the scratch's error word: no bounded wait ran out


def test_noalloc_qwen_layer_batch1_twice():
    W = synth.layer_weights(synth.QWEN3_30B_A3B, seed=0, device="cuda")
    layer = M.Layer(W, top_e=8).build_sketch(synth.rot_seed(0)).build_lowrank(32)
    st = layer.struct()
    for s in range(2):
        x = synth.tokens(2048, 1, seed=40 + s).cuda()
        ref = layer.forward(x, k=136, c=272)
        y = torch.empty_like(x)
        M.moe_reader_forward_noalloc(st, 1, 136, 272, x, None, y)
        torch.cuda.synchronize()
        _close(y, ref)
    M.moe_reader_check_error(None)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """B = 256 on the Qwen layer shape needs more than the 8 MiB scratch: the
    call is refused by validation, before anything is enqueued (the pointers
    below are never dereferenced)."""
    fake = 0x10000
    st = M.MoeReaderLayer(E=128, I=768, d=2048, top_e=8, r=32, w_router=fake, router_bias=None, w_gate=fake,
                          w_up=fake, w_down=fake, rot_sign=fake, sk_gate=fake, sk_up=fake, alpha_gate=fake,
                          alpha_up=fake, u_sigma=fake, v=fake)
    assert M.moe_reader_workspace_bytes(256, 128, 8, 768, 2048, 136, 272, 32) > 8 << 20
    with pytest.raises(M.MoeError, match="MOE_EINVAL.*workspace"):
        M.moe_reader_forward_noalloc(st, 256, 136, 272, fake, None, fake)
