"""Failure detection on the GPU without a GPU fault: every device wait on a
bulk copy is bounded, and a wait that runs out records an error word instead
of hanging.  A test hook of the forward call withholds one sketch copy of
each work item of the one-cluster reader and shortens the wait limit to a
millisecond: the kernel completes (its outputs are unusable), the error word
reads MOE_ETIMEOUT, and the same workspace then runs a normal step that
matches the oracle (the context stays usable).

Read before running (the kernel side): after a wait runs out the reader goes
on through every remaining stage; every cluster barrier is reached by every
CTA unconditionally, the withheld copy was never issued (nothing is left in
flight into shared memory), and the later waits on the same barrier run out
after the same short limit."""
import pytest
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from tests.gpu_helpers import OracleCache, check_pair

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B", [1, 2])
def test_withheld_copy_times_out_and_the_next_step_is_clean(B):
    W = synth.layer_weights(synth.TINY, seed=0)
    seed = synth.rot_seed(0)
    layer = M.Layer(W, top_e=2).build_sketch(seed)
    oc = OracleCache(W, seed, 8)
    layer.path = 1  # the one-cluster reader
    x = synth.tokens(256, B, seed=70).cuda()
    ws = layer.workspace(B)
    y = torch.empty_like(x)
    layer.set_lowrank(None, None)
    dbg = M.MoeReaderDebug()
    dbg.wait_limit_us = 1000
    dbg.withhold_copy = 1
    M.moe_reader_forward(layer.struct(), B, 24, 48, x, None, y, dbg, ws, ws.numel())
    with pytest.raises(M.MoeError, match="MOE_ETIMEOUT"):
        layer.check()
    # the error word was cleared by the check; a normal step on the same
    # workspace is correct and leaves it clear
    M.moe_reader_check_error(ws)
    check_pair(layer, oc, synth.tokens(256, B, seed=71), k=24, c=48, top_e=2)
    M.moe_reader_check_error(ws)
