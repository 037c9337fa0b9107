"""GPU parity of both readers where the automatic choice does not take
them: the streamed kernels at one and two tokens, the one-cluster reader at
pinned cluster sizes, and the two paths against each other.  The reader is
chosen per call (the layer's `path` field), so two threads that ask for
different readers at the same time each get their own."""
import threading

import numpy as np
import pytest
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from tests.gpu_helpers import OracleCache, bf16_ulp, check_pair

pytestmark = pytest.mark.gpu

QWEN = synth.QWEN3_30B_A3B
AUTO, CLUSTER, STREAMED = 0, 1, 2


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


class using:
    """Sets a layer's reader path and cluster size for the block."""

    def __init__(self, layer, path=AUTO, cluster_size=0):
        self.layer, self.path, self.cs = layer, path, cluster_size

    def __enter__(self):
        self.layer.path, self.layer.cluster_size = self.path, self.cs
        return self.layer

    def __exit__(self, *exc):
        self.layer.path, self.layer.cluster_size = AUTO, 0


@pytest.mark.parametrize("B", [1, 2])
@pytest.mark.parametrize("recovery_input", [0, 1])
def test_streamed_tiny_small_batch(tiny, B, recovery_input):
    _, layer, oc = tiny
    with using(layer, STREAMED):
        for seed in range(3):
            check_pair(layer, oc, synth.tokens(256, B, seed=seed), k=24, c=48, top_e=2, recovery_input=recovery_input)


@pytest.mark.parametrize("k,c,r", [(1, 1, 8), (128, 128, 0), (5, 17, 0), (64, 100, 8)])
def test_streamed_tiny_budgets_batch1(tiny, k, c, r):
    W, layer, _ = tiny
    oc = OracleCache(W, synth.rot_seed(0), r)
    with using(layer, STREAMED):
        check_pair(layer, oc, synth.tokens(256, 1, seed=12), k=k, c=c, top_e=2)


@pytest.mark.parametrize("recovery_input", [0, 1])
def test_streamed_qwen_batch1(qwen, recovery_input):
    _, layer, oc = qwen
    with using(layer, STREAMED):
        for seed in (0, 7):
            check_pair(layer, oc, synth.tokens(2048, 1, seed=seed), k=136, c=272, top_e=8,
                       recovery_input=recovery_input)


@pytest.mark.parametrize("cs", [2, 4, 6, 8])
@pytest.mark.parametrize("B", [1, 2])
def test_cluster_reader_pinned_sizes_tiny(tiny, cs, B):
    """Other channel and column partitions of the one-cluster reader (the
    automatic size differs), with every exact-stage slot count they give."""
    _, layer, oc = tiny
    with using(layer, CLUSTER, cs):
        check_pair(layer, oc, synth.tokens(256, B, seed=60 + cs), k=24, c=48, top_e=2)


@pytest.mark.parametrize("cs", [6, 8, 16])
def test_cluster_reader_pinned_sizes_qwen(qwen, cs):
    """Six CTAs own 128 channels each (exact rows in several rounds per
    warp), sixteen own 48: both ends of the partition at the layer shape."""
    _, layer, oc = qwen
    with using(layer, CLUSTER, cs):
        check_pair(layer, oc, synth.tokens(2048, 1, seed=80 + cs), k=136, c=272, top_e=8)
        check_pair(layer, oc, synth.tokens(2048, 2, seed=90 + cs), k=136, c=272, top_e=8)


@pytest.mark.parametrize("B", [1, 2])
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
            out[p] = layer.forward(x, k=136, c=272, debug=True, path=p)
            layer.check()
    finally:
        layer.set_lowrank(None, None)
    (y1, d1), (y2, d2) = out[CLUSTER], out[STREAMED]
    for n in ("ids", "dot_gate", "dot_up", "cand"):
        assert torch.equal(d1[n], d2[n]), n
    assert torch.equal(d1["score"].view(torch.int32), d2["score"].view(torch.int32))
    k1, k2 = d1["kept"].cpu().numpy(), d2["kept"].cpu().numpy()
    assert (k1 == k2).mean() > 0.99  # near-tie swaps of |a| only
    a, b = y1.float().cpu().numpy(), y2.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2 * bf16_ulp(np.maximum(np.abs(a), np.abs(b))) + 1e-3)


def test_two_threads_get_their_own_reader(qwen):
    """Two host threads run steps at the same time, one asking for the
    one-cluster reader and one for the streamed reader (separate layers'
    descriptors, workspaces and streams).  Each gets the reader it asked for:
    only the one-cluster reader writes stage time stamps."""
    _, layer, _ = qwen
    x = synth.tokens(2048, 1, seed=5).cuda()
    lay2 = M.Layer.__new__(M.Layer)
    lay2.__dict__.update(layer.__dict__)
    lay2._ws = None  # its own workspace
    res = {}

    def run(lay, p):
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            for _ in range(20):
                _, dbg = lay.forward(x, k=136, c=272, debug=True, path=p, stream=s)
            s.synchronize()
        res[p] = int((dbg["phase_ns"].cpu() != 0).sum())

    th = [threading.Thread(target=run, args=(layer, CLUSTER)), threading.Thread(target=run, args=(lay2, STREAMED))]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert res[CLUSTER] > 0 and res[STREAMED] == 0, res
