"""The expert-parallel exchange on CPU: two gloo ranks each take the experts
e % 2 == rank, form their partial of the block from the oracle's per-slot
outputs, and call ep_step (one all-reduce, then the finish).  Every rank must
end with the oracle's whole block, rounded once to bf16."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from calibration_free_channel_b200 import ep, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    from oracle import oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = synth.layer_weights(synth.TINY, seed=0)
        sk = O.build_sketch(W["w_gate"], W["w_up"], synth.rot_seed(0))
        lr = O.build_lowrank(W["w_down"], 8)
        x = synth.tokens(256, 3, seed=7)
        res = synth.tokens(256, 3, seed=8)
        yb, y64, od = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, residual=res, debug=True)
        owned = (od["ids"] % world) == rank
        part = np.einsum("bs,bsd->bd", np.where(owned, od["weights"], 0.0).astype(np.float64), od["y_expert"])
        partial = torch.from_numpy(part).float()
        resf = torch.from_numpy(O.bf16_to_f64(res)).float()
        y = ep.ep_step(partial, lambda ys: (ys + resf).to(torch.bfloat16))
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(y64), 2.0 ** -126))) - 7)
        err = np.abs(y.double().numpy() - y64)
        out[rank] = float((err / ulp).max())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_ep_step_gloo_matches_whole_block(world):
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert sorted(out.keys()) == list(range(world))
    # each rank holds the whole block: within one bf16 ulp of the fp64 output
    assert all(v <= 1.0 for v in out.values()), dict(out)


def test_owned_experts_partition():
    E = 128
    for world in (1, 2, 3, 8):
        parts = [ep.owned_experts(E, r, world) for r in range(world)]
        flat = sorted(e for p in parts for e in p)
        assert flat == list(range(E))
        assert all(len(p) in (E // world, E // world + 1) for p in parts)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_weights_holds_only_owned_experts(world):
    """ep.shard_weights: the router whole, the experts e % world == rank
    stacked in order, and the slot map the C layer's expert_slot takes."""
    W = synth.layer_weights(synth.TINY, seed=0, bias=True)
    E = W["w_router"].shape[0]
    seen = []
    for rank in range(world):
        Wr, slot = ep.shard_weights(W, rank, world)
        own = ep.owned_experts(E, rank, world)
        assert torch.equal(Wr["w_router"], W["w_router"]) and torch.equal(Wr["router_bias"], W["router_bias"])
        for n in ("w_gate", "w_up", "w_down"):
            assert Wr[n].shape[0] == len(own)
            assert torch.equal(Wr[n], W[n][own])
        assert slot.dtype == torch.int32 and slot.shape == (E,)
        assert slot[own].tolist() == list(range(len(own)))
        assert all(int(slot[e]) == -1 for e in range(E) if e not in own)
        seen += own
    assert sorted(seen) == list(range(E))
