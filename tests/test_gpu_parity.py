"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded inputs, on the tiny block, the Qwen3-30B-A3B-shaped layer at
batch 1, the budget and batch sweeps, and edge cases."""
import numpy as np
import pytest
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from oracle import oracle as O
from tests.gpu_helpers import MAX_ABS, REL_L2, OracleCache, bf16_ulp, check_pair

pytestmark = pytest.mark.gpu

QWEN = synth.QWEN3_30B_A3B


@pytest.fixture(scope="module")
def tiny():
    W = synth.layer_weights(synth.TINY, seed=0)
    seed = synth.rot_seed(0)
    layer = M.Layer(W, top_e=2).build_sketch(seed)
    return W, layer, OracleCache(W, seed, 8)


@pytest.fixture(scope="module")
def qwen():
    W = synth.layer_weights(QWEN, seed=0)
    seed = synth.rot_seed(0)
    layer = M.Layer(W, top_e=8).build_sketch(seed)
    return W, layer, OracleCache(W, seed, 32)


@pytest.fixture(scope="module")
def qwen_skewed():
    W = synth.layer_weights(QWEN, seed=1, bias=True)
    seed = synth.rot_seed(1)
    layer = M.Layer(W, top_e=8).build_sketch(seed)
    return W, layer, OracleCache(W, seed, 32)


# ------------------------------------------------------------------ sketch
def _check_sketch(layer, oc):
    s, skg, sku, ag, au = oc.sk
    assert np.array_equal(layer.rot_sign.cpu().numpy(), s)
    assert np.array_equal(layer.sk_gate.cpu().numpy().view(np.uint32), skg)
    assert np.array_equal(layer.sk_up.cpu().numpy().view(np.uint32), sku)
    assert np.array_equal(layer.alpha_gate.cpu().numpy().view(np.uint32), ag.view(np.uint32))
    assert np.array_equal(layer.alpha_up.cpu().numpy().view(np.uint32), au.view(np.uint32))


def test_build_sketch_bit_exact_tiny(tiny):
    _, layer, oc = tiny
    _check_sketch(layer, oc)


def test_build_sketch_bit_exact_qwen_layer(qwen):
    _, layer, oc = qwen
    _check_sketch(layer, oc)


# ---------------------------------------------------------------- forward
@pytest.mark.parametrize("B", [1, 2, 5])
def test_forward_tiny(tiny, B):
    W, layer, oc = tiny
    for seed in range(3):
        x = synth.tokens(256, B, seed=seed)
        check_pair(layer, oc, x, k=24, c=48, top_e=2)


@pytest.mark.parametrize("k,c,r", [(1, 1, 8), (24, 24, 8), (24, 128, 8), (128, 128, 0), (5, 17, 0), (64, 100, 8)])
def test_forward_tiny_budgets(tiny, k, c, r):
    W, layer, _ = tiny
    oc = OracleCache(W, synth.rot_seed(0), r)
    x = synth.tokens(256, 3, seed=11)
    if r == 0:
        layer.set_lowrank(None, None)
    check_pair(layer, oc, x, k=k, c=c, top_e=2)


def test_forward_qwen_layer_batch1_steps(qwen):
    """The Qwen3-30B-A3B-shaped layer at batch 1 over all 20 decode steps
    (tokens from seeds 0..19; k = 136, c = 272, r = 32)."""
    W, layer, oc = qwen
    for s in range(20):
        x = synth.tokens(2048, 1, seed=s)
        check_pair(layer, oc, x, k=136, c=272, top_e=8)


@pytest.mark.parametrize("B", [1, 4, 8, 16])
@pytest.mark.parametrize("k", [100, 136])
def test_forward_qwen_budget_sweep(qwen, B, k):
    """The budget sweep: k = 100 (13%) and k = 136 (18%), c = 2k, r = 32, at
    batch 1, 4, 8 and 16 (tokens drawn independently)."""
    W, layer, oc = qwen
    x = synth.tokens(2048, B, seed=100 + B + k)
    check_pair(layer, oc, x, k=k, c=2 * k, top_e=8)


@pytest.mark.parametrize("B", [1, 8, 16, 32, 64])
def test_forward_qwen_skewed_batch(qwen_skewed, B):
    """Skewed router prior (logit bias ~ N(0, 1) per expert), the batch sweep
    at 1, 8, 16, 32 and 64 tokens: at the larger batches many tokens share
    experts, so one expert's tokens span several work items."""
    W, layer, oc = qwen_skewed
    x = synth.tokens(2048, B, seed=200 + B)
    _, ids, _ = O.route(x, W["w_router"], W["router_bias"], 8)
    if B >= 32:
        assert np.bincount(ids.ravel()).max() > 8
    check_pair(layer, oc, x, k=136, c=272, top_e=8)


def test_forward_with_own_lowrank_build(qwen):
    """End to end with the GPU's own sketch and low-rank map against the
    oracle's own (both built from the weights alone)."""
    W, layer, oc = qwen
    layer.build_lowrank(32)
    x = synth.tokens(2048, 2, seed=300)
    check_pair(layer, oc, x, k=136, c=272, top_e=8, use_oracle_factors=False)


def test_identical_tokens_share_work_items(tiny):
    W, layer, oc = tiny
    x1 = synth.tokens(256, 1, seed=5)
    x = x1.repeat(11, 1)  # 11 tokens on the same 2 experts: items of 8 + 3
    check_pair(layer, oc, x, k=24, c=48, top_e=2)


@pytest.mark.parametrize("B,pinned", [(1, True), (1, False), (16, True)])
def test_forward_host_matches_forward(qwen, B, pinned):
    """The host-buffer entry equals the device one bit for bit: pinned buffers
    go through the copy kernels, pageable ones through cudaMemcpyAsync."""
    W, layer, oc = qwen
    x = synth.tokens(2048, B, seed=7)
    y_dev = layer.forward(x.cuda(), k=136, c=272)
    xh = x.pin_memory() if pinned else x.clone()
    yh = torch.empty_like(xh).pin_memory() if pinned else torch.empty_like(xh)
    xd = torch.empty_like(x, device="cuda")
    yd = torch.empty_like(x, device="cuda")
    ws = layer.workspace(B)
    M.moe_reader_forward_host(layer.struct(), B, 136, 272, xh, xd, yd, yh, ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())


# ------------------------------------------------------------------ dense
def _check_out(y, y64):
    yg = y.float().cpu().numpy().astype(np.float64)
    assert (np.abs(yg - y64) - 0.5 * bf16_ulp(y64)).max() <= MAX_ABS
    assert np.linalg.norm(yg - y64) / np.linalg.norm(y64) <= REL_L2


@pytest.mark.parametrize("B", [1, 9])
def test_dense_tiny(tiny, B):
    W, layer, _ = tiny
    x = synth.tokens(256, B, seed=20 + B)
    y = layer.forward_dense(x.cuda())
    _, y64 = O.forward_dense(x, W, top_e=2)
    _check_out(y, y64)


def test_dense_qwen_layer(qwen):
    W, layer, _ = qwen
    x = synth.tokens(2048, 2, seed=21)
    y = layer.forward_dense(x.cuda())
    _, y64 = O.forward_dense(x, W, top_e=8)
    _check_out(y, y64)


def test_all_channels_kept_equals_dense_on_gpu(qwen):
    """k = c = I with recovery off is the dense block (property, any size)."""
    W, layer, _ = qwen
    x = synth.tokens(2048, 3, seed=22).cuda()
    ys = layer.forward(x, k=768, c=768, r=0).float()
    yd = layer.forward_dense(x).float()
    ulp = torch.from_numpy(bf16_ulp(yd.cpu().numpy())).cuda()
    assert ((ys - yd).abs() - 2 * ulp).max().item() <= MAX_ABS
    assert ((ys - yd).norm() / yd.norm()).item() <= REL_L2


# ------------------------------------------ recovery from the exact a of dropped candidates
@pytest.mark.parametrize("B", [1, 2, 5])
def test_forward_recovery_exact_input_tiny(tiny, B):
    W, layer, oc = tiny
    for seed in range(2):
        x = synth.tokens(256, B, seed=40 + seed)
        check_pair(layer, oc, x, k=24, c=48, top_e=2, recovery_input=1)


@pytest.mark.parametrize("B", [1, 4])
def test_forward_recovery_exact_input_qwen(qwen, B):
    W, layer, oc = qwen
    x = synth.tokens(2048, B, seed=50 + B)
    check_pair(layer, oc, x, k=136, c=272, top_e=8, recovery_input=1)


@pytest.mark.parametrize("k", [1, 24, 77])
def test_recovery_exact_input_all_candidates_exact_map_equals_dense_on_gpu(tiny, k):
    """c = I, exact full-rank map (Ubar = I, V = W_down^T): with the exact
    recovery input every skipped channel comes back exactly, so the reader
    equals the dense block for every k (a property that holds at any size)."""
    W, layer, oc = tiny
    E, I = 8, 128
    eye = torch.zeros((E, I, I), dtype=torch.float32)
    eye[:, torch.arange(I), torch.arange(I)] = 1.0
    vt = W["w_down"].transpose(1, 2).contiguous()
    layer.set_lowrank(eye.to(torch.bfloat16), vt)
    try:
        x = synth.tokens(256, 3, seed=60).cuda()
        ys = layer.forward(x, k=k, c=I, recovery_input=1).float()
        yd = layer.forward_dense(x).float()
        ulp = torch.from_numpy(bf16_ulp(yd.cpu().numpy())).cuda()
        assert ((ys - yd).abs() - 2 * ulp).max().item() <= MAX_ABS
        assert ((ys - yd).norm() / yd.norm()).item() <= REL_L2
        # the default recovery input (sketch estimates) does not come back exactly
        y0 = layer.forward(x, k=k, c=I, recovery_input=0).float()
        assert ((y0 - yd).norm() / yd.norm()).item() > 5 * REL_L2
    finally:
        layer.set_lowrank(None, None)


# ---------------------------------------------------------------- lowrank
def _lowrank_check(W, layer, r, experts):
    us = layer.u_sigma.float().cpu().numpy()
    vv = layer.v.float().cpu().numpy()
    wd = synth.bf16_bits(W["w_down"])
    for e in experts:
        ubar, V, S = O.lowrank_f64(wd[e], r)
        want = ubar @ V.T
        got = us[e].astype(np.float64) @ vv[e].astype(np.float64).T
        assert np.linalg.norm(got - want) <= 1e-2 * np.linalg.norm(want)
        # sign rule (applied before the bf16 rounding): the largest positive
        # entry of each v column is within one bf16 ulp of its largest magnitude
        for p in range(r):
            col = vv[e][:, p].astype(np.float64)
            top = np.abs(col).max()
            assert col.max() >= top - bf16_ulp(top)
        # residual close to the optimum (Eckart-Young)
        Wf = O.bf16_to_f64(wd[e])
        best = np.sqrt(max(np.sum(S[r:] ** 2), 0))
        assert np.linalg.norm(Wf - got) <= best * 1.01 + 1e-6 * np.linalg.norm(Wf)


def test_build_lowrank_tiny(tiny):
    W, layer, _ = tiny
    layer.build_lowrank(8)
    _lowrank_check(W, layer, 8, range(8))


def test_build_lowrank_qwen_layer(qwen):
    W, layer, _ = qwen
    layer.build_lowrank(32)
    _lowrank_check(W, layer, 32, [0, 17, 64, 127])


# ---------------------------------------------------------------- rmsnorm
def test_rmsnorm_matches_oracle():
    x = synth.tokens(2048, 5, seed=3)
    x = (x.float() * 3.7).to(torch.bfloat16)
    h = torch.empty_like(x, device="cuda")
    M.moe_reader_rmsnorm(5, 2048, 1e-6, x.cuda(), h)
    torch.cuda.synchronize()
    ho = O.rmsnorm(x)
    diff = np.abs(O.bf16_to_f64(h.cpu()) - O.bf16_to_f64(ho))
    assert diff.max() <= 2 ** -7 * np.abs(O.bf16_to_f64(ho)).max()
