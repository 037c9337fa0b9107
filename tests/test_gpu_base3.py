"""Base-3 sketch rows on the GPU (five trits per byte): the repacked bytes
against the oracle's packing of the oracle's trits, and both readers' sketch
dots, scores and candidate sets against the oracle, bit for bit, when they
decode base-3 rows ("KAIST: MoE Decoding Needs No Calibration Data", section
"A reader that needs no data at all": the resident sketch is about 7% of the
BF16 checkpoint; 2-bit codes are 8.3%, five trits per byte 6.8%)."""
import numpy as np
import pytest

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from oracle import oracle as O
from tests.gpu_helpers import OracleCache, check_pair

pytestmark = pytest.mark.gpu

QWEN = synth.QWEN3_30B_A3B


def _trits_of_codes(words, d):
    """Trits of rows of 2-bit code words (position 4p + b of a word at bits
    8b + 2p as the code T + 1), decoded independently of both builders."""
    j = np.arange(16)
    shift = 8 * (j & 3) + 2 * (j >> 2)
    codes = (words[..., None].astype(np.uint64) >> shift.astype(np.uint64)) & 3
    return (codes.reshape(words.shape[:-1] + (d,)).astype(np.int16) - 1).astype(np.int8)


def _check_bytes(layer, oc, experts):
    d = layer.d
    rb = M.moe_reader_sketch_row_bytes(d, 1)
    nb = (d + 4) // 5
    _, skg, sku, _, _ = oc.sk
    for gpu, ora in ((layer.sk_gate, skg), (layer.sk_up, sku)):
        g = gpu.cpu().numpy()
        assert g.shape == (layer.E, layer.I, rb)
        assert (g[..., nb:] == 121).all()  # sector padding: five zero trits per byte
        for e in experts:
            t = _trits_of_codes(ora[e], d)
            want = np.stack([O.pack_trits_base3(t[i]) for i in range(layer.I)])
            assert np.array_equal(g[e, :, :nb], want)
            back = np.stack([O.unpack_trits_base3(np.ascontiguousarray(g[e, i, :nb]), d) for i in range(layer.I)])
            assert np.array_equal(back, t)


@pytest.fixture(scope="module")
def tiny3():
    W = synth.layer_weights(synth.TINY, seed=0)
    seed = synth.rot_seed(0)
    return W, M.Layer(W, top_e=2).build_sketch(seed, packing="base3"), OracleCache(W, seed, 8)


@pytest.fixture(scope="module")
def qwen3():
    W = synth.layer_weights(QWEN, seed=0)
    seed = synth.rot_seed(0)
    return W, M.Layer(W, top_e=8).build_sketch(seed, packing="base3"), OracleCache(W, seed, 32)


def test_base3_bytes_tiny(tiny3):
    _, layer, oc = tiny3
    _check_bytes(layer, oc, range(layer.E))


def test_base3_bytes_qwen_layer(qwen3):
    _, layer, oc = qwen3
    _check_bytes(layer, oc, (0, 63, 127))


@pytest.mark.parametrize("B,path", [(1, 1), (2, 1), (1, 2), (5, 0), (16, 0)])
def test_base3_parity_tiny(tiny3, B, path):
    W, layer, oc = tiny3
    layer.path = path
    try:
        for s in range(3):
            x = synth.tokens(256, B, seed=300 + 10 * B + s)
            check_pair(layer, oc, x, k=24, c=48, top_e=2)
    finally:
        layer.path = 0


@pytest.mark.parametrize("B", [1, 2, 16])
def test_base3_parity_qwen_layer(qwen3, B):
    W, layer, oc = qwen3
    for s in range(2):
        x = synth.tokens(QWEN.d, B, seed=500 + 10 * B + s)
        check_pair(layer, oc, x, k=136, c=272, top_e=8)


def test_base3_d4096_streamed():
    """d = 4096 (two 80-trit chunk lanes per part in the streamed screen)."""
    shape = synth.BlockShape(E=8, I=128, d=4096, top_e=2)
    W = synth.layer_weights(shape, seed=2)
    seed = synth.rot_seed(2)
    layer = M.Layer(W, top_e=2).build_sketch(seed, packing="base3")
    oc = OracleCache(W, seed, 8)
    _check_bytes(layer, oc, (0, 7))
    for B in (1, 3):
        check_pair(layer, oc, synth.tokens(4096, B, seed=700 + B), k=24, c=48, top_e=2)
