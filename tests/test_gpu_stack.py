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


# ------------------------------------------------------ 48-layer stack (config 4)
def _oracle_parts(Wh, experts, rot_seed, r, lowrank=True):
    """The oracle's sketch and low-rank factors of one layer, built from its
    weights for the given experts only (the rest stay zero and are never
    read): the sketch rows of those experts, and (lowrank) their rank-r SVD
    maps, several SVDs at a time."""
    from concurrent.futures import ThreadPoolExecutor
    E, I, d = Wh["w_gate"].shape
    experts = sorted(set(int(e) for e in np.ravel(experts)))
    s = np.empty(d, np.int8)
    skg = np.zeros((E, I, d // 16), np.uint32)
    sku = np.zeros_like(skg)
    ag = np.zeros((E, I), np.float32)
    au = np.zeros_like(ag)
    sub = O.build_sketch(Wh["w_gate"][experts], Wh["w_up"][experts], rot_seed)
    s[:] = sub[0]
    skg[experts], sku[experts], ag[experts], au[experts] = sub[1], sub[2], sub[3], sub[4]
    if not lowrank:
        return (s, skg, sku, ag, au), None
    wd = synth.bf16_bits(Wh["w_down"])
    us = np.zeros((E, I, r), np.uint16)
    vv = np.zeros((E, d, r), np.uint16)
    with ThreadPoolExecutor(8) as ex:
        for e, (ubar, V, _) in zip(experts, ex.map(lambda e: O.lowrank_f64(wd[e], r), experts)):
            us[e] = O.f64_to_bf16(ubar)
            vv[e] = O.f64_to_bf16(V)
    return (s, skg, sku, ag, au), (us, vv)


@pytest.mark.slow
def test_stack_48_layers_cold_decode():
    """Config 4: a 48-layer stack of Qwen3-30B-A3B-shaped blocks (about 58 GB
    of bf16 expert weights, independent seeded weights per layer, drawn on the
    device), x_{l+1} = x_l + MoE_l(RMSNorm(x_l)), k = 136, c = 272, r = 32,
    the GPU's own sketches and low-rank maps.
      - At batch 1 and batch 16 the first, a middle and the last layer are
        checked against the oracle on the GPU's own layer input (teacher
        forcing; the oracle builds its sketch from the weights for the
        experts it routes to, and reads the layer's low-rank factors as every
        parity test gives both sides the same factors: two bf16-rounded
        rank-32 maps from different SVD methods differ enough to move a
        per-expert output by 2e-2, and the builders have tests of their
        own).
      - At batch 1 the oracle also runs the first four layers on its own
        activations: the GPU's output stays within 5e-2 relative L2 of it.
        Further on, the two free runs decorrelate on these random weights: a
        near-tie routing or kept-set choice, or the last bits of the two
        low-rank builds, changes one layer's output and the residual stream
        carries it to every later layer.  So after 48 layers only the
        activations are checked to stay finite and of bounded scale."""
    shape, L, k, c, r, top = synth.QWEN3_30B_A3B, 48, 136, 272, 32, 8
    layers = []
    for l in range(L):
        W = synth.layer_weights(shape, seed=0, layer=l, device="cuda")
        layers.append(M.Layer(W, top_e=top).build_sketch(synth.rot_seed(0, l)).build_lowrank(r))
    torch.cuda.synchronize()
    checked, free_layers = (0, L // 2, L - 1), 4
    for B, tok_seed in ((1, 41), (16, 42)):
        x = synth.tokens(shape.d, B, seed=tok_seed).cuda()
        x_free = synth.bf16_bits(x.cpu())
        for l, lay in enumerate(layers):
            h = torch.empty_like(x)
            M.moe_reader_rmsnorm(B, shape.d, EPS, x, h)
            y, dbg = lay.forward(h, k=k, c=c, residual=x, debug=True)
            lay.check()
            free = B == 1 and l < free_layers
            Wh = {n: (v.cpu() if v is not None else None) for n, v in lay.w.items()} if l in checked or free \
                else None
            if l in checked:
                hb = h.cpu()
                logits, ids, _ = O.route(hb, Wh["w_router"], None, top)
                sk, _ = _oracle_parts(Wh, ids, synth.rot_seed(0, l), r, lowrank=False)
                lr = (lay.u_sigma.view(torch.int16).cpu().numpy().view(np.uint16),
                      lay.v.view(torch.int16).cpu().numpy().view(np.uint16))
                _, y64, odbg = O.forward(hb, Wh, sk, lr, k=k, c=c, r=r, top_e=top,
                                         residual=synth.bf16_bits(x.cpu()), debug=True)
                compare_step(Wh, hb, y, dbg, y64, odbg, k, ora_logits=logits)
            if free:
                hf = O.rmsnorm(x_free, EPS)
                _, idf, _ = O.route(hf, Wh["w_router"], None, top)
                skf, lrf = _oracle_parts(Wh, idf, synth.rot_seed(0, l), r)
                x_free, _, _ = O.forward(hf, Wh, skf, lrf, k=k, c=c, r=r, top_e=top, residual=x_free)
                if l == free_layers - 1:
                    yg, yf = O.bf16_to_f64(y.cpu()), O.bf16_to_f64(x_free)
                    drift = np.linalg.norm(yg - yf) / np.linalg.norm(yf)
                    assert drift < 5e-2, (l, drift)
            x = y
        yg = O.bf16_to_f64(x.cpu())
        x0 = O.bf16_to_f64(synth.tokens(shape.d, B, seed=tok_seed))
        assert np.isfinite(yg).all()
        # each layer adds one block output of about the input's scale
        assert np.linalg.norm(yg) < 4 * np.sqrt(L) * np.linalg.norm(x0)
    del layers
    torch.cuda.empty_cache()
