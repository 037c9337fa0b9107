"""Read accounting in 32-byte sectors: the analytic count equals a brute-force
set of touched sector addresses ("KAIST: MoE Decoding Needs No Calibration
Data", section "Calibrated thresholds do not pin down how much you read": a
sector touched at all is billed in full)."""
import numpy as np

from calibration_free_channel_b200 import accounting, synth
from oracle import oracle as O


def _bruteforce_sectors(E, I, d, r, ids, cand, kept, bias):
    base = {}
    nxt = 0
    sizes = dict(w_router=E * d * 2, bias=E * 4, sk_gate=E * I * d // 4, sk_up=E * I * d // 4,
                 alpha_gate=E * I * 4, alpha_up=E * I * 4, w_gate=E * I * d * 2, w_up=E * I * d * 2,
                 w_down=E * I * d * 2, u_sigma=E * I * r * 2, v=E * d * r * 2)
    for n, sz in sizes.items():
        base[n] = nxt
        nxt += (sz + 255) // 256 * 256 + 4096
    touched = set()

    def read(name, off, nbytes):
        a = base[name] + off
        touched.update(range(a // 32, (a + nbytes - 1) // 32 + 1))

    read("w_router", 0, E * d * 2)
    if bias:
        read("bias", 0, E * 4)
    for e in np.unique(ids):
        for nm in ("sk_gate", "sk_up"):
            for i in range(I):
                read(nm, (e * I + i) * d // 4, d // 4)
        for nm in ("alpha_gate", "alpha_up"):
            read(nm, e * I * 4, I * 4)
        bs, ss = np.nonzero(ids == e)
        for b, s in zip(bs, ss):
            for i in cand[b, s]:
                read("w_gate", (e * I + i) * d * 2, d * 2)
                read("w_up", (e * I + i) * d * 2, d * 2)
            for i in kept[b, s]:
                # the down rows are read in column slices; the slices tile the row
                for j0 in range(0, d, d // 16):
                    read("w_down", (e * I + i) * d * 2 + j0 * 2, d // 16 * 2)
        if r:
            read("u_sigma", e * I * r * 2, I * r * 2)
            read("v", e * d * r * 2, d * r * 2)
    return len(touched) * 32


def test_sector_count_matches_bruteforce():
    shape = synth.TINY
    W = synth.layer_weights(shape, seed=0, bias=True)
    sk = O.build_sketch(W["w_gate"], W["w_up"], 3)
    lr = O.build_lowrank(W["w_down"], 8)
    x = synth.tokens(256, 4, seed=2)
    _, _, dbg = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, debug=True)
    acc = accounting.step_bytes(8, 128, 256, 8, dbg["ids"], dbg["cand"], dbg["kept"], bias=True)
    assert acc["total"] == _bruteforce_sectors(8, 128, 256, 8, dbg["ids"], dbg["cand"], dbg["kept"], True)


def test_fixed_budget_numbers_of_the_qwen3_layer():
    # one token, 8 experts, k = 136, c = 272, r = 32
    assert accounting.expert_bytes(768, 2048, 32, 272, 136)["total"] == 3_758_080
    assert accounting.fixed_budget_step_bytes(128, 768, 2048, 32, 136, 272, 8) == 30_588_928
    assert accounting.expert_bytes(768, 2048, 32, 200, 100)["total"] == 3_020_800
    assert accounting.router_bytes(128, 2048, False) + 8 * accounting.dense_expert_bytes(768, 2048) == 76_021_760


def test_top_k_read_budget_is_input_independent():
    """Top-k fixes how much is read: every token reads the same bytes."""
    shape = synth.TINY
    W = synth.layer_weights(shape, seed=1)
    sk = O.build_sketch(W["w_gate"], W["w_up"], 4)
    totals = set()
    for seed in range(6):
        x = synth.tokens(256, 1, seed=seed)
        _, _, dbg = O.forward(x, W, sk, None, k=24, c=48, r=0, top_e=2, debug=True)
        totals.add(accounting.step_bytes(8, 128, 256, 0, dbg["ids"], dbg["cand"], dbg["kept"])["total"])
    assert len(totals) == 1


def test_expert_bytes_with_base3_sketch_rows():
    # the Qwen layer shape: sketch rows of 416 bytes instead of 512, the rest unchanged
    two = accounting.expert_bytes(768, 2048, 32, 272, 136)
    three = accounting.expert_bytes(768, 2048, 32, 272, 136, packing="base3")
    assert two["sketch"] == 2 * 768 * 512 + 2 * 768 * 4 == 792576
    assert three["sketch"] == 2 * 768 * 416 + 2 * 768 * 4 == 645120
    assert two["total"] - three["total"] == two["sketch"] - three["sketch"]
    assert three["total"] % accounting.SECTOR == 0
