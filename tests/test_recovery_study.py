"""Output error of the reader against the dense block, as a function of the
budget k, the candidate count c, the rank r and the recovery input.

"KAIST: MoE Decoding Needs No Calibration Data", section "A reader that needs
no data at all": skipped channels are recovered through a low-rank map of the
down projections.  Two inputs to that map are compared:
  recovery_input = 0: sketch estimates a-hat for every channel outside the
                      kept set (the plain reading);
  recovery_input = 1: the exact a for candidates that were computed but not
                      kept, a-hat only outside the candidate set.
The error is rel-L2 of the fp64 block output against the dense SwiGLU block
on the same routing, averaged over tokens.  The assertions hold with margin on
the synthetic recipe; running this file as a script prints the table on the
Qwen3-30B-A3B layer shape (python -m tests.test_recovery_study)."""
import numpy as np
import pytest

from calibration_free_channel_b200 import synth
from oracle import oracle as O

SHAPE = synth.BlockShape(E=16, I=768, d=2048, top_e=8)


def setup(shape, n_tok, seed=0, layer=5, r_max=32):
    W = synth.layer_weights(shape, seed=seed, layer=layer)
    sk = O.build_sketch(W["w_gate"], W["w_up"], synth.rot_seed(seed, layer))
    toks = [synth.tokens(shape.d, 1, seed=3000 + s) for s in range(n_tok)]
    used = set()
    for x in toks:
        used |= set(O.route(x, W["w_router"], None, shape.top_e)[1].ravel().tolist())
    lr = {r: O.build_lowrank(W["w_down"], r, experts=sorted(used)) for r in {r_max, 8}}
    dense = [O.forward_dense(x, W, top_e=shape.top_e)[1] for x in toks]
    return W, sk, toks, lr, dense


def rel_err(ctx, shape, k, c, r, recovery_input):
    W, sk, toks, lr, dense = ctx
    errs = []
    for x, yd in zip(toks, dense):
        _, y, _ = O.forward(x, W, sk, lr[r] if r else None, k=k, c=c, r=r, top_e=shape.top_e,
                            recovery_input=recovery_input)
        errs.append(np.linalg.norm(y - yd) / np.linalg.norm(yd))
    return np.asarray(errs)


@pytest.fixture(scope="module")
def ctx():
    return setup(SHAPE, n_tok=3)


def test_exact_input_beats_sketch_input(ctx):
    # with the exact a of dropped candidates the recovery no longer adds the
    # sketch's error on the largest skipped channels
    for k in (100, 136):
        e0 = rel_err(ctx, SHAPE, k, 2 * k, 32, 0)
        e1 = rel_err(ctx, SHAPE, k, 2 * k, 32, 1)
        assert e1.mean() < e0.mean(), (k, e0, e1)


def test_error_falls_with_budget(ctx):
    e = [rel_err(ctx, SHAPE, k, 2 * k, 32, 1).mean() for k in (64, 136, 272)]
    assert e[0] > e[1] > e[2], e


def test_no_dropped_candidates_makes_the_inputs_agree(ctx):
    # c = k: every candidate is kept, so the two recovery inputs are the same
    W, sk, toks, lr, _ = ctx
    for x in toks[:2]:
        y0 = O.forward(x, W, sk, lr[32], k=136, c=136, r=32, top_e=SHAPE.top_e, recovery_input=0)[1]
        y1 = O.forward(x, W, sk, lr[32], k=136, c=136, r=32, top_e=SHAPE.top_e, recovery_input=1)[1]
        assert np.array_equal(y0, y1)


def main(shape=synth.QWEN3_30B_A3B, n_tok=4):
    ctx = setup(shape, n_tok)
    print("| k | c | r | recovery input | rel-L2 vs dense (mean, min-max) |")
    print("|---|---|---|---|---|")
    for k in (100, 136, 200):
        for c in (k, 2 * k):
            for r, ri in ((0, 0), (8, 1), (32, 0), (32, 1)):
                if c == k and ri == 1:
                    continue
                e = rel_err(ctx, shape, k, c, r, ri)
                name = "-" if r == 0 else ("exact a of dropped candidates" if ri else "a-hat")
                print(f"| {k} | {c} | {r} | {name} | {e.mean():.4f} ({e.min():.4f}-{e.max():.4f}) |",
                      flush=True)


if __name__ == "__main__":
    main()
