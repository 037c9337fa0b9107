"""GPU parity of the expert-parallel step (moe_reader_forward_ep +
moe_reader_ep_finish).  The ranks are emulated one after another on one GPU:
each rank's launches are independent (no rank waits on another), and the
all-reduce of the partials is a plain sum here.  Every rank's partial is
checked against the oracle's sum over the slots it owns, and the finished
output against the oracle's whole block."""
import numpy as np
import pytest
import torch

from calibration_free_channel_b200 import moe_reader as M
from calibration_free_channel_b200 import synth
from oracle import oracle as O
from tests.gpu_helpers import MAX_ABS, REL_L2, OracleCache, bf16_ulp

pytestmark = pytest.mark.gpu

QWEN = synth.QWEN3_30B_A3B


@pytest.fixture(scope="module")
def tiny():
    W = synth.layer_weights(synth.TINY, seed=0)
    seed = synth.rot_seed(0)
    return W, M.Layer(W, top_e=2).build_sketch(seed), OracleCache(W, seed, 8), 2


@pytest.fixture(scope="module")
def qwen():
    W = synth.layer_weights(QWEN, seed=0)
    seed = synth.rot_seed(0)
    return W, M.Layer(W, top_e=8).build_sketch(seed), OracleCache(W, seed, 32), 8


def _run(fixture, world, B, k, c, seed, recovery_input=0):
    W, layer, oc, top_e = fixture
    d = W["w_gate"].shape[2]
    x = synth.tokens(d, B, seed=seed)
    _, ids, _ = O.route(x, W["w_router"], None, top_e)
    lr = oc.lowrank_for(ids)
    layer.set_lowrank(torch.from_numpy(lr[0].view(np.int16)).view(torch.bfloat16),
                      torch.from_numpy(lr[1].view(np.int16)).view(torch.bfloat16))
    _, y64, od = O.forward(x, W, oc.sk, lr, k=k, c=c, r=oc.r, top_e=top_e, debug=True,
                           recovery_input=recovery_input)
    xd = x.cuda()
    parts = []
    for rank in range(world):
        yp, g = layer.forward_ep(xd, k, c, rank, world, debug=True, recovery_input=recovery_input)
        layer.check()
        g = {n: v.cpu().numpy() for n, v in g.items()}
        assert np.array_equal(g["ids"], od["ids"]), "routing differs"
        owned = (od["ids"] % world) == rank
        # owned pairs: candidate sets bit-exact, kept sets equal on these seeds
        assert np.array_equal(g["cand"][owned], od["cand"][owned])
        # the rank's partial against the oracle's over its slots (fp32 outputs)
        want = np.einsum("bs,bsd->bd", np.where(owned, od["weights"], 0.0).astype(np.float64), od["y_expert"])
        got = yp.cpu().numpy().astype(np.float64)
        kept_ok = all(set(g["kept"][b, s]) == set(od["kept"][b, s]) for b, s in zip(*np.nonzero(owned)))
        if kept_ok:
            assert np.abs(got - want).max() <= MAX_ABS, f"rank {rank}: partial error {np.abs(got - want).max()}"
        parts.append(yp)
    y_sum = torch.stack(parts).sum(0)  # the all-reduce
    y = torch.empty_like(xd)
    M.moe_reader_ep_finish(B, d, y_sum, None, y)
    yv = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(yv - y64)
    assert np.all(err <= bf16_ulp(y64) + MAX_ABS), err.max()
    assert np.linalg.norm(yv - y64) <= REL_L2 * np.linalg.norm(y64)
    layer.set_lowrank(None, None)
    return y


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("B", [1, 5])
def test_ep_tiny(tiny, world, B):
    _run(tiny, world, B, k=24, c=48, seed=31 + B)


@pytest.mark.parametrize("world", [2, 8])
def test_ep_qwen_layer(qwen, world):
    _run(qwen, world, B=4, k=136, c=272, seed=41)


def test_ep_qwen_layer_exact_recovery_input(qwen):
    _run(qwen, 4, B=2, k=136, c=272, seed=42, recovery_input=1)


def test_ep_finish_adds_residual_and_rounds_once():
    B, d = 3, 256
    y_sum = torch.randn(B, d, dtype=torch.float32, device="cuda")
    res = synth.tokens(d, B, seed=5).cuda()
    y = torch.empty_like(res)
    M.moe_reader_ep_finish(B, d, y_sum, res, y)
    want = (y_sum.double() + res.double()).float().to(torch.bfloat16)  # one rounding of the fp32 sum
    assert torch.equal(y.view(torch.int16), want.view(torch.int16))


def test_ep_rejects_bad_rank(tiny):
    _, layer, _, _ = tiny
    x = synth.tokens(256, 1, seed=0).cuda()
    with pytest.raises(M.MoeError):
        layer.forward_ep(x, 24, 48, 2, 2)


@pytest.mark.parametrize("world", [2, 8])
def test_compacted_shards_match_the_full_layer(qwen, world):
    """A rank that holds only its experts (compacted [E/N, ...] arrays and
    expert_slot) computes the same partial, bit for bit, as a rank that
    holds the whole layer, and holds 1/N of the expert bytes."""
    W, layer, oc, top_e = qwen
    x = synth.tokens(QWEN.d, 4, seed=43).cuda()
    full_bytes = sum(t.numel() * t.element_size() for t in (layer.w["w_gate"], layer.w["w_up"], layer.w["w_down"],
                                                          layer.sk_gate, layer.sk_up))
    for rank in range(world):
        S = layer.shard(rank, world)
        held = sum(t.numel() * t.element_size() for t in (S.w["w_gate"], S.w["w_up"], S.w["w_down"], S.sk_gate,
                                                        S.sk_up))
        assert S.w["w_gate"].shape[0] == len(range(rank, QWEN.E, world))
        assert held * world == full_bytes
        want = layer.forward_ep(x, 136, 272, rank, world)
        got = S.forward_ep(x, 136, 272, rank, world)
        layer.check()
        S.check()
        assert torch.equal(got, want)


def test_compacted_shard_base3_sketch(tiny):
    """The slot indirection also covers base-3 sketch rows."""
    W, _, _, _ = tiny
    full = M.Layer(W, top_e=2).build_sketch(synth.rot_seed(0), packing="base3").build_lowrank(8)
    x = synth.tokens(256, 5, seed=44).cuda()
    for rank in range(2):
        want = full.forward_ep(x, 24, 48, rank, 2)
        got = full.shard(rank, 2).forward_ep(x, 24, 48, rank, 2)
        assert torch.equal(got, want)


def test_forward_with_a_missing_expert_reports_edevice(tiny):
    """A plain step whose routing reaches an expert with no weight slot reads
    slot 0 in its place (in bounds) and reports MOE_EDEVICE; the next check
    is clean."""
    W, layer, _, _ = tiny
    S = layer.shard(0, 2)  # holds experts 0, 2, 4, 6 only
    x = synth.tokens(256, 8, seed=45).cuda()  # 8 tokens x 2 slots reach odd experts too
    S.forward(x, k=24, c=48)
    with pytest.raises(M.MoeError, match="MOE_EDEVICE"):
        S.check()
    S.check()


def test_shard_weights_builds_the_same_rank(tiny):
    """A rank built from only its experts' weights (ep.shard_weights, never
    holding the others) equals the slice of the full layer."""
    from calibration_free_channel_b200 import ep
    W, layer, _, _ = tiny
    Wr, slot = ep.shard_weights(W, 1, 2)
    R = M.Layer(Wr, top_e=2, expert_slot=slot).build_sketch(synth.rot_seed(0)).build_lowrank(8)
    S = M.Layer(W, top_e=2).build_sketch(synth.rot_seed(0)).build_lowrank(8).shard(1, 2)
    assert torch.equal(R.sk_gate, S.sk_gate) and torch.equal(R.u_sigma, S.u_sigma)
    x = synth.tokens(256, 3, seed=46).cuda()
    assert torch.equal(R.forward_ep(x, 24, 48, 1, 2), S.forward_ep(x, 24, 48, 1, 2))
