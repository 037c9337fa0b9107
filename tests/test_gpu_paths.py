"""GPU parity of both readers at batch sizes where the automatic choice does
not take them: the streamed kernels at one and two tokens, the one-cluster
kernel above two tokens, and the two paths against each other."""
import numpy as np
import pytest
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from tests.gpu_helpers import OracleCache, bf16_ulp, check_pair

pytestmark = pytest.mark.gpu

QWEN = synth.QWEN3_30B_A3B
CLUSTER, STREAMED = 1, 2


@pytest.fixture(scope="module")
def tiny():
    W = synth.layer_weights(synth.TINY, seed=0)
    seed = synth.rot_seed(0)
    return W, M.Layer(W, top_e=2).build_sketch(seed), OracleCache(W, seed, 8)


@pytest.fixture(scope="module")
def qwen():
    W = synth.layer_weights(QWEN, seed=0)
    seed = synth.rot_seed(0)
    return W, M.Layer(W, top_e=8).build_sketch(seed), OracleCache(W, seed, 32)


@pytest.fixture
def path(request):
    M.moe_reader_set_path(request.param)
    try:
        yield request.param
    finally:
        M.moe_reader_set_path(0)


@pytest.mark.parametrize("path", [STREAMED], indirect=True)
@pytest.mark.parametrize("B", [1, 2])
@pytest.mark.parametrize("recovery_input", [0, 1])
def test_streamed_tiny_small_batch(tiny, path, B, recovery_input):
    _, layer, oc = tiny
    for seed in range(3):
        check_pair(layer, oc, synth.tokens(256, B, seed=seed), k=24, c=48, top_e=2, recovery_input=recovery_input)


@pytest.mark.parametrize("path", [STREAMED], indirect=True)
@pytest.mark.parametrize("k,c,r", [(1, 1, 8), (128, 128, 0), (5, 17, 0), (64, 100, 8)])
def test_streamed_tiny_budgets_batch1(tiny, path, k, c, r):
    W, layer, _ = tiny
    oc = OracleCache(W, synth.rot_seed(0), r)
    check_pair(layer, oc, synth.tokens(256, 1, seed=12), k=k, c=c, top_e=2)


@pytest.mark.parametrize("path", [STREAMED], indirect=True)
@pytest.mark.parametrize("recovery_input", [0, 1])
def test_streamed_qwen_batch1(qwen, path, recovery_input):
    _, layer, oc = qwen
    for seed in (0, 7):
        check_pair(layer, oc, synth.tokens(2048, 1, seed=seed), k=136, c=272, top_e=8, recovery_input=recovery_input)


@pytest.mark.parametrize("path", [CLUSTER], indirect=True)
@pytest.mark.parametrize("B", [3, 4])
def test_cluster_path_above_two_tokens(tiny, qwen, path, B):
    _, lt, ot = tiny
    check_pair(lt, ot, synth.tokens(256, B, seed=40 + B), k=24, c=48, top_e=2)
    _, lq, oq = qwen
    check_pair(lq, oq, synth.tokens(2048, B, seed=50 + B), k=136, c=272, top_e=8)


@pytest.mark.parametrize("B", [1, 3, 16])
def test_paths_agree(qwen, B):
    """Routing, sketch dots, scores and candidate sets agree bit for bit
    between the two readers; kept sets agree; outputs agree to the rounding
    of the exact stage's summation order (one bf16 ulp plus a little)."""
    _, layer, oc = qwen
    x = synth.tokens(2048, B, seed=70 + B).cuda()
    layer.build_lowrank(32)  # both paths read the same factors
    out = {}
    try:
        for p in (CLUSTER, STREAMED):
            M.moe_reader_set_path(p)
            out[p] = layer.forward(x, k=136, c=272, debug=True)
            layer.check()
    finally:
        M.moe_reader_set_path(0)
        layer.set_lowrank(None, None)
    (y1, d1), (y2, d2) = out[CLUSTER], out[STREAMED]
    for n in ("ids", "dot_gate", "dot_up", "cand"):
        assert torch.equal(d1[n], d2[n]), n
    assert torch.equal(d1["score"].view(torch.int32), d2["score"].view(torch.int32))
    k1, k2 = d1["kept"].cpu().numpy(), d2["kept"].cpu().numpy()
    assert (k1 == k2).mean() > 0.99  # near-tie swaps of |a| only
    a, b = y1.float().cpu().numpy(), y2.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2 * bf16_ulp(np.maximum(np.abs(a), np.abs(b))) + 1e-3)
