"""GPU parity of the residual path and of a stack of MoE blocks (the cold-cache
decode step through several layers): x_{l+1} = x_l + MoE_l(RMSNorm(x_l)).

Each layer is checked with teacher forcing: the oracle takes the GPU's own
layer input x_l, so a layer's comparison does not inherit the rounding of the
layers before it.  The end-to-end drift of an oracle run on its own
activations is checked separately against a loose bound."""
import numpy as np
import pytest
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from oracle import oracle as O
from tests.gpu_helpers import OracleCache, bf16_ulp, compare_step

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _layer(shape, seed, layer, top_e, r):
    W = synth.layer_weights(shape, seed=seed, layer=layer)
    rs = synth.rot_seed(seed, layer)
    return W, M.Layer(W, top_e=top_e).build_sketch(rs), OracleCache(W, rs, r)


def _step_gpu(lay, oc, x, k, c, top_e):
    """One block on the GPU: h = RMSNorm(x), x' = x + MoE(h); the oracle's
    low-rank factors are loaded so both sides read identical inputs."""
    B, d = x.shape
    h = torch.empty_like(x)
    M.moe_reader_rmsnorm(B, d, EPS, x, h)
    _, ids, _ = O.route(h.cpu(), oc.W["w_router"], oc.W.get("router_bias"), top_e)
    lr = oc.lowrank_for(ids)
    lay.set_lowrank(torch.from_numpy(lr[0].view(np.int16)).view(torch.bfloat16),
                    torch.from_numpy(lr[1].view(np.int16)).view(torch.bfloat16))
    y, dbg = lay.forward(h, k=k, c=c, residual=x, debug=True)
    lay.check()
    return h, y, dbg, lr


@pytest.mark.parametrize("B", [1, 3])
def test_residual_matches_oracle_tiny(B):
    W, lay, oc = _layer(synth.TINY, 0, 0, 2, 8)
    x = synth.tokens(256, B, seed=11)
    res = synth.tokens(256, B, seed=12)
    logits, ids, _ = O.route(x, W["w_router"], None, 2)
    lr = oc.lowrank_for(ids)
    lay.set_lowrank(torch.from_numpy(lr[0].view(np.int16)).view(torch.bfloat16),
                    torch.from_numpy(lr[1].view(np.int16)).view(torch.bfloat16))
    y, dbg = lay.forward(x.cuda(), k=24, c=48, residual=res.cuda(), debug=True)
    _, y64, odbg = O.forward(x, W, oc.sk, lr, k=24, c=48, r=8, top_e=2, residual=res, debug=True)
    compare_step(W, x, y, dbg, y64, odbg, 24, ora_logits=logits)
    # the residual is really added: without it the output moves by the residual
    y0, _ = lay.forward(x.cuda(), k=24, c=48, debug=True)
    yv, y0v = y.float().cpu().numpy(), y0.float().cpu().numpy()
    # each output is rounded once to bf16: the difference is the residual up to two roundings
    tol = bf16_ulp(yv) + bf16_ulp(y0v)
    assert np.all(np.abs((yv - y0v) - O.bf16_to_f64(res)) <= tol)


def _stack(shape, L, B, k, c, top_e, r, seed, tok_seed):
    layers = [_layer(shape, seed, l, top_e, r) for l in range(L)]
    x = synth.tokens(shape.d, B, seed=tok_seed).cuda()
    x_free = synth.bf16_bits(x.cpu())  # the oracle's own run, no teacher forcing
    for l, (W, lay, oc) in enumerate(layers):
        h, y, dbg, lr = _step_gpu(lay, oc, x, k, c, top_e)
        xb = synth.bf16_bits(x.cpu())
        # RMSNorm of the GPU's layer input, against the oracle's
        ho = O.bf16_to_f64(O.rmsnorm(xb, EPS))
        hg = O.bf16_to_f64(h.cpu())
        assert np.abs(hg - ho).max() <= 2 ** -7 * np.abs(ho).max(), f"layer {l}: rmsnorm"
        # the block, teacher-forced on the GPU's h and x
        logits, _, _ = O.route(h.cpu(), W["w_router"], None, top_e)
        _, y64, odbg = O.forward(h.cpu(), W, oc.sk, lr, k=k, c=c, r=r, top_e=top_e, residual=xb, debug=True)
        compare_step(W, h.cpu(), y, dbg, y64, odbg, k, ora_logits=logits)
        # the oracle's free run through the same layer
        hf = O.rmsnorm(x_free, EPS)
        _, idf, _ = O.route(hf, W["w_router"], None, top_e)
        x_free, _, _ = O.forward(hf, W, oc.sk, oc.lowrank_for(idf), k=k, c=c, r=r, top_e=top_e, residual=x_free)
        x = y
    yg = O.bf16_to_f64(x.cpu())
    yf = O.bf16_to_f64(x_free)
    drift = np.linalg.norm(yg - yf) / np.linalg.norm(yf)
    return drift


def test_stack_tiny_four_layers():
    drift = _stack(synth.TINY, L=4, B=2, k=24, c=48, top_e=2, r=8, seed=0, tok_seed=21)
    # bf16 rounding compounds through the residual stream; a routing flip on a
    # near-tie may change one expert of one layer, so the bound is loose
    assert drift < 5e-2, drift


def test_stack_qwen_layer_shape_two_layers_batch1():
    drift = _stack(synth.QWEN3_30B_A3B, L=2, B=1, k=136, c=272, top_e=8, r=32, seed=0, tok_seed=22)
    assert drift < 5e-2, drift
