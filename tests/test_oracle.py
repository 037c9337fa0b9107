"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these re-type the oracle's formulas: each checks a closed form, an
invariant, a library routine on a special case, a hand-derived fixture or a
brute force on tiny inputs.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from calibration_free_channel_b200 import synth
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(a):
    return synth.bf16_bits(torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def f32_ulp_diff(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


# ----------------------------------------------------------------- SplitMix64
def test_splitmix64_published_outputs():
    lines = [l for l in open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt")) if not l.startswith("#")]
    want = [int(l) for l in lines if l.strip()]
    got = [O.splitmix64_at(1234567, j) for j in range(len(want))]
    assert got == want


def test_rot_signs_are_pm1_and_balanced():
    s = O.rot_signs(1 << 14, 42)
    assert set(np.unique(s)) == {-1, 1}
    assert abs(float(s.mean())) < 0.05
    assert not np.array_equal(O.rot_signs(64, 1), O.rot_signs(64, 2))


# ---------------------------------------------------------------------- FWHT
@pytest.mark.parametrize("d", [2, 8, 64, 256])
def test_fwht_equals_sylvester_hadamard_on_integers(d):
    rng = np.random.default_rng(d)
    v = rng.integers(-50, 50, d).astype(np.float32)
    got = O.fwht(v).astype(np.float64)
    want = scipy.linalg.hadamard(d).astype(np.float64) @ v.astype(np.float64)
    assert np.array_equal(got, want)


def test_fwht_involution_and_parseval():
    rng = np.random.default_rng(1)
    v = rng.integers(-1000, 1000, 2048).astype(np.float32)
    assert np.array_equal(O.fwht(O.fwht(v)), v * 2048)  # H H = d I, exact on integers
    x = rng.standard_normal(2048).astype(np.float32)
    y = O.fwht(x).astype(np.float64)
    assert abs(np.dot(y, y) - 2048 * np.dot(x.astype(np.float64), x)) < 1e-4 * 2048 * np.dot(x, x)


# ------------------------------------------------------------------ exp / SiLU
def test_exp_r_within_2ulp_of_exact_exp():
    ts = np.concatenate([np.linspace(-87, 88, 20001), np.linspace(-1, 1, 5001), [0.0, 1e-8, -1e-8]])
    ts = ts.astype(np.float32)
    got = np.array([O.exp_r(t) for t in ts], np.float32)
    want = np.array([math.exp(float(t)) for t in ts]).astype(np.float32)  # correctly rounded enough
    assert f32_ulp_diff(got, want).max() <= 2
    assert O.exp_r(0.0) == 1.0


def test_exp_r_clamps_to_normal_range():
    assert O.exp_r(-1000.0) == O.exp_r(-87.0) > 0
    assert np.isfinite(O.exp_r(1000.0)) and O.exp_r(1000.0) == O.exp_r(88.0)
    assert O.exp_r(-87.0) >= np.finfo(np.float32).tiny


def test_silu_r_matches_fp64_silu_and_identity():
    ts = np.linspace(-30, 30, 6001).astype(np.float32)
    got = np.array([O.silu_r(t) for t in ts])
    want = ts.astype(np.float64) / (1 + np.exp(-ts.astype(np.float64)))
    assert np.all(np.abs(got - want) <= 4e-7 * np.maximum(np.abs(want), 1e-30) + 1e-37)
    # silu(t) - silu(-t) = t
    neg = np.array([O.silu_r(-t) for t in ts])
    assert np.allclose(got - neg, ts, rtol=1e-6, atol=1e-6)
    assert O.silu_r(0.0) == 0.0


# ------------------------------------------------------------ closed forms
def _parse_sparse(spec, d=16):
    v = np.zeros(d, np.float32)
    for tok in spec.split():
        val, idx = tok.split("@")
        v[int(idx)] = float(val)
    return v


def _parse_signs(spec, d=16):
    s = np.ones(d, np.int8)
    for tok in spec.split():
        if "@" in tok:
            s[int(tok.split("@")[1])] = -1
    return s


def _golden_cases(kind):
    for line in open(os.path.join(GOLDEN, "closed_forms.txt")):
        if line.startswith("#") or not line.strip():
            continue
        head, signs, inp, exp = [p.strip() for p in line.split("|")]
        k, name = head.split()
        if k == kind:
            yield name, _parse_signs(signs), _parse_sparse(inp), dict(t.split("=") for t in exp.split())


@pytest.mark.parametrize("case", list(_golden_cases("twn")), ids=lambda c: c[0])
def test_twn_hand_derived(case):
    name, s, w, exp = case
    trits, alpha, _ = O.twn_row(bf16(w), s)
    want = [{"+": 1, "-": -1, "0": 0}[ch] for ch in exp["trits"]]
    assert trits.tolist() == want
    assert alpha == float(exp["alpha"])


def _expand(spec):
    out = []
    for part in spec.split(","):
        if "x" in part:
            v, n = part.split("x")
            out += [int(v)] * int(n)
        else:
            out.append(int(part))
    return out


@pytest.mark.parametrize("case", list(_golden_cases("quant")), ids=lambda c: c[0])
def test_quantize_hand_derived(case):
    name, s, x, exp = case
    v, q, cx = O.rotate_quantize(bf16(x)[None, :][0], s)
    want = _expand(exp["q"])
    if len(want) < 16:  # "a,bxN" alternates a at even, b at odd indices
        a, b = want[0], want[1]
        want = [a if m % 2 == 0 else b for m in range(16)]
    assert q.tolist() == want
    num, _, den = exp["cx"].partition("/")
    assert cx == np.float32(float(num) / float(den)) if den else cx == float(num)


def test_quantize_error_bound_and_range():
    rng = np.random.default_rng(3)
    s = O.rot_signs(2048, 7)
    for _ in range(5):
        x = bf16(rng.standard_t(4, 2048))
        v, q, cx = O.rotate_quantize(x, s)
        amax = np.abs(v).max()
        assert np.abs(q).max() == 127
        deq = q.astype(np.float64) * amax / 127
        assert np.all(np.abs(deq - v) <= amax / 254 * (1 + 1e-6))
        assert np.isclose(cx, amax / (127 * 2048), rtol=1e-7)
        # v = H (s x): Sylvester Hadamard from scipy, fp64
        xf = O.bf16_to_f64(x)
        want = scipy.linalg.hadamard(2048) @ (s * xf)
        assert np.allclose(v, want, rtol=0, atol=1e-5 * np.abs(want).max())


# ---------------------------------------------------------------- packing
def _independent_unpack(words, d):
    """Decoder written from the documented layout, vectorised differently:
    for each byte b and pair p, the 2-bit field at bits 8b + 2p is the code
    of position 4p + b."""
    w = np.asarray(words, np.uint64)
    out = np.zeros((w.size, 16), np.int64)
    for b in range(4):
        for p in range(4):
            code = (w >> np.uint64(8 * b + 2 * p)) & np.uint64(3)
            assert not np.any(code == 3)
            out[:, 4 * p + b] = code.astype(np.int64) - 1
    return out.reshape(-1)[:d]


def test_pack_roundtrip_and_layout():
    rng = np.random.default_rng(5)
    t = rng.integers(-1, 2, 256).astype(np.int8)
    p = O.pack_trits(t)
    assert np.array_equal(_independent_unpack(p, 256), t)
    zero = np.zeros(16, np.int8)
    assert O.pack_trits(zero)[0] == 0x55555555  # every code 01 (T = 0)
    one = zero.copy()
    one[9] = -1  # position 9 = 4*2 + 1: byte 1, pair 2 -> bits [12, 13] = 00
    assert O.pack_trits(one)[0] == 0x55555555 & ~(3 << 12)
    one = zero.copy()
    one[3] = 1  # position 3 = 4*0 + 3: byte 3, pair 0 -> bits [24, 25] = 10
    assert O.pack_trits(one)[0] == (0x55555555 & ~(3 << 24)) | (2 << 24)
    # a masked word times four int8 activations, minus their sum, is the dot
    q = rng.integers(-127, 128, 16)
    w = int(O.pack_trits(t[:16])[0])
    acc = 0
    for pp in range(4):
        m = (w >> (2 * pp)) & 0x03030303
        acc += sum(((m >> (8 * b)) & 0xFF) * q[4 * pp + b] for b in range(4))
    assert acc - q.sum() == int(np.dot(t[:16].astype(np.int64), q))


# ---------------------------------------------------------------- sketch
@pytest.fixture(scope="module")
def tiny():
    W = synth.layer_weights(synth.TINY, seed=0)
    sk = O.build_sketch(W["w_gate"], W["w_up"], synth.rot_seed(0))
    lr = O.build_lowrank(W["w_down"], 8)
    return W, sk, lr


def test_sketch_is_weight_only_and_deterministic(tiny):
    W, sk, _ = tiny
    sk2 = O.build_sketch(W["w_gate"], W["w_up"], synth.rot_seed(0))
    for a, b in zip(sk, sk2):
        assert np.array_equal(a, b)


def test_twn_alpha_is_least_squares_scale_and_threshold_separates(tiny):
    W, sk, _ = tiny
    s = sk[0]
    wg = synth.bf16_bits(W["w_gate"])
    for row in range(0, 128, 17):
        t, alpha, wrot = O.twn_row(wg[0, row], s)
        wr = wrot.astype(np.float64)
        err = lambda a: np.sum((wr - a * t) ** 2)
        assert err(alpha) <= min(err(alpha * 1.01), err(alpha * 0.99))
        nz = t != 0
        assert np.all(np.sign(wr[nz]) == t[nz])
        assert np.abs(wr[~nz]).max() < np.abs(wr[nz]).min()
        assert np.isclose(np.abs(wr[nz]).min() if nz.any() else 0, np.abs(wr[nz]).min())


def test_sketch_dots_are_exact_integers(tiny):
    W, sk, lr = tiny
    x = synth.tokens(256, 1, seed=3)
    _, _, dbg = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, debug=True)
    _, q, _ = O.rotate_quantize(synth.bf16_bits(x)[0], sk[0])
    for s in range(2):
        e = dbg["ids"][0, s]
        T = _independent_unpack(sk[1][e].reshape(-1), 128 * 256).reshape(128, 256)
        assert np.array_equal(T @ q.astype(np.int64), dbg["dot_gate"][0, s])
        T = _independent_unpack(sk[2][e].reshape(-1), 128 * 256).reshape(128, 256)
        assert np.array_equal(T @ q.astype(np.int64), dbg["dot_up"][0, s])


def test_sketch_estimates_track_exact_dots():
    """alpha * c_x * (T.q) estimates W.x (H^T H = d I); a wrong scale (a lost
    1/d, a dropped c_x or alpha) breaks the ratio."""
    shape = synth.BlockShape(E=1, I=256, d=1024, top_e=1)
    W = synth.layer_weights(shape, seed=1)
    s, skg, sku, ag, au = O.build_sketch(W["w_gate"], W["w_up"], 11)
    x = synth.tokens(1024, 1, seed=1)
    _, q, cx = O.rotate_quantize(synth.bf16_bits(x)[0], s)
    T = _independent_unpack(skg[0].reshape(-1), 256 * 1024).reshape(256, 1024)
    est = (T @ q.astype(np.float64)) * ag[0] * cx
    exact = O.bf16_to_f64(W["w_gate"][0]) @ O.bf16_to_f64(x)[0]
    assert np.corrcoef(est, exact)[0, 1] > 0.8
    slope = np.dot(est, exact) / np.dot(exact, exact)
    assert 0.8 < slope < 1.25


# ---------------------------------------------------------------- router
def test_router_topk_bruteforce_and_weights():
    shape = synth.BlockShape(E=16, I=16, d=256, top_e=4)
    W = synth.layer_weights(shape, seed=2, bias=True)
    x = synth.tokens(256, 3, seed=2)
    logits, ids, w = O.route(x, W["w_router"], W["router_bias"], top_e=4)
    want = O.bf16_to_f64(x) @ O.bf16_to_f64(W["w_router"]).T + W["router_bias"].numpy().astype(np.float64)
    assert np.allclose(logits, want, rtol=1e-12, atol=1e-12)
    for b in range(3):
        order = sorted(range(16), key=lambda e: (-want[b, e], e))[:4]
        assert ids[b].tolist() == order
        full = np.exp(want[b] - want[b].max())
        full /= full.sum()
        ren = full[order] / full[order].sum()  # softmax over all, keep top, renormalise
        assert np.allclose(w[b], ren, rtol=1e-6)
        assert abs(w[b].sum() - 1) < 1e-6


def test_router_ties_go_to_lower_id():
    wr = np.zeros((8, 256), np.float32)
    wr[:, 0] = [1, 3, 3, 2, 3, 0, 0, 0]
    x = np.zeros((1, 256), np.float32)
    x[0, 0] = 1
    _, ids, w = O.route(bf16(x), bf16(wr), None, top_e=3)
    assert ids[0].tolist() == [1, 2, 4]
    assert np.allclose(w[0], 1 / 3)


# ---------------------------------------------------------------- selection
def test_top_n_bruteforce_subsets_with_ties():
    rng = np.random.default_rng(9)
    for trial in range(30):
        keys = rng.integers(0, 6, 12).astype(np.float32)  # many ties
        got = O.top_n(keys, 3)
        best = max(itertools.combinations(range(12), 3),
                   key=lambda S: (sum(keys[list(S)]), [-i for i in sorted(S)]))
        # among maximal-sum subsets, lower indices win ties
        assert got.tolist() == sorted(best)


def test_expert_top_k_is_exhaustive_optimum_tiny():
    """I = 12 channels, c = I, k = 3: the kept set maximises sum |a| over all
    220 subsets, with a computed here in fp64 (gap checked)."""
    rng = np.random.default_rng(4)
    I, d = 12, 16
    wg = bf16(rng.standard_normal((1, I, d)) * 0.3)
    wu = bf16(rng.standard_normal((1, I, d)) * 0.3)
    wd = bf16(rng.standard_normal((1, I, d)) * 0.3)
    W = dict(w_router=bf16(rng.standard_normal((1, d))), w_gate=wg, w_up=wu, w_down=wd, router_bias=None)
    x = bf16(rng.standard_normal((1, d)))
    sk = O.build_sketch(wg, wu, 5)
    _, _, dbg = O.forward(x, W, sk, None, k=3, c=I, r=0, top_e=1, debug=True)
    xf = O.bf16_to_f64(x)[0]
    g = O.bf16_to_f64(wg[0]) @ xf
    u = O.bf16_to_f64(wu[0]) @ xf
    a = np.abs(g / (1 + np.exp(-g)) * u)
    srt = np.sort(a)[::-1]
    assert srt[2] - srt[3] > 1e-4 * srt[2]
    best = max(itertools.combinations(range(I), 3), key=lambda S: a[list(S)].sum())
    assert dbg["kept"][0, 0].tolist() == sorted(best)
    assert dbg["cand"][0, 0].tolist() == list(range(I))


# ------------------------------------------------------------ invariants
def _dense_numpy(x, W, top_e):
    """Dense SwiGLU MoE written with numpy matmuls (fp64)."""
    logits, ids, w = O.route(x, W["w_router"], W.get("router_bias"), top_e)
    xf = O.bf16_to_f64(x)
    y = np.zeros_like(xf)
    for b in range(xf.shape[0]):
        for s in range(top_e):
            e = ids[b, s]
            g = O.bf16_to_f64(W["w_gate"][e]) @ xf[b]
            u = O.bf16_to_f64(W["w_up"][e]) @ xf[b]
            y[b] += w[b, s] * (O.bf16_to_f64(W["w_down"][e]).T @ (g / (1 + np.exp(-g)) * u))
    return y


def test_dense_oracle_matches_numpy_matmul(tiny):
    W, _, _ = tiny
    x = synth.tokens(256, 2, seed=5)
    _, y64 = O.forward_dense(x, W, top_e=2)
    assert np.allclose(y64, _dense_numpy(x, W, 2), rtol=1e-10, atol=1e-12)


def test_invariant_all_channels_no_recovery_equals_dense(tiny):
    """(i) k = I with recovery off is the dense SwiGLU expert."""
    W, sk, _ = tiny
    x = synth.tokens(256, 2, seed=6)
    _, y64, _ = O.forward(x, W, sk, None, k=128, c=128, r=0, top_e=2)
    _, yd = O.forward_dense(x, W, top_e=2)
    assert np.abs(y64 - yd).max() <= 1e-5 * np.abs(yd).max()


@pytest.mark.parametrize("k", [1, 24, 77, 128])
def test_invariant_exact_sketch_full_rank_map_equals_dense(tiny, k):
    """(ii) With exact screening values and an exact full-rank map
    (Ubar = I_I, V = W_down^T, so Ubar V^T = W_down in bf16), the reader
    equals the dense expert for every k: kept channels are read, the rest
    are recovered exactly."""
    W, sk, _ = tiny
    E, I, d = 8, 128, 256
    us = np.zeros((E, I, I), np.uint16)
    us[:, np.arange(I), np.arange(I)] = bf16(np.ones(1))[0]
    vv = np.ascontiguousarray(np.transpose(synth.bf16_bits(W["w_down"]), (0, 2, 1)))
    x = synth.tokens(256, 2, seed=7)
    _, y64, dbg = O.forward(x, W, sk, (us, vv), k=k, c=min(2 * k, I), r=I, top_e=2, exact_mode=True,
                            debug=True)
    _, yd = O.forward_dense(x, W, top_e=2)
    assert np.abs(y64 - yd).max() <= 1e-5 * np.abs(yd).max()
    # and without recovery the error is large unless k = I
    _, y0, _ = O.forward(x, W, sk, None, k=k, c=min(2 * k, I), r=0, top_e=2, exact_mode=True)
    if k < I:
        assert np.abs(y0 - yd).max() > 1e-3 * np.abs(yd).max()


@pytest.mark.parametrize("k", [1, 24, 77])
def test_recovery_variant_all_candidates_exact_map_equals_dense(tiny, k):
    """Recovery variant with every channel a candidate (c = I): each skipped
    channel enters the map with its exact a, so with the exact full-rank map
    (Ubar = I, V = W_down^T) the block equals the dense one for every k,
    without the exact-sketch test mode.  The default input (sketch estimates
    for the skipped channels) does not."""
    W, sk, _ = tiny
    E, I, d = 8, 128, 256
    x = synth.tokens(d, 2, seed=8)
    eye = O.f64_to_bf16(np.broadcast_to(np.eye(I), (E, I, I)).copy())
    wdT = np.ascontiguousarray(np.transpose(synth.bf16_bits(W["w_down"]), (0, 2, 1)))
    yd = O.forward_dense(x, W, top_e=2)[1]
    _, yv, _ = O.forward(x, W, sk, (eye, wdT), k=k, c=I, r=I, top_e=2, recovery_input=1)
    assert np.abs(yv - yd).max() <= 1e-5 * np.abs(yd).max()
    _, y0, _ = O.forward(x, W, sk, (eye, wdT), k=k, c=I, r=I, top_e=2, recovery_input=0)
    assert not np.allclose(y0, yd, rtol=0, atol=1e-3 * np.abs(yd).max())


def test_recovery_variant_equals_default_in_exact_sketch_mode(tiny):
    """With exact screening estimates (ahat = a for every channel) the two
    recovery inputs are the same numbers."""
    W, sk, lr = tiny
    x = synth.tokens(256, 2, seed=9)
    _, ya, _ = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, exact_mode=True, recovery_input=0)
    _, yb, _ = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, exact_mode=True, recovery_input=1)
    assert np.array_equal(ya, yb)


def test_invariant_svd_full_rank_map_equals_dense(tiny):
    """(ii) with the SVD map at full rank r = I (factors rounded to bf16)."""
    W, sk, _ = tiny
    lr = O.build_lowrank(W["w_down"], 128)
    x = synth.tokens(256, 1, seed=8)
    _, y64, _ = O.forward(x, W, sk, lr, k=24, c=48, r=128, top_e=2, exact_mode=True)
    _, yd = O.forward_dense(x, W, top_e=2)
    assert np.linalg.norm(y64 - yd) <= 2e-2 * np.linalg.norm(yd)


def test_invariant_exactly_k_kept_c_candidates(tiny):
    """(iii) top-k keeps exactly k per (token, expert), whatever the input."""
    W, sk, lr = tiny
    x = synth.tokens(256, 4, seed=9)
    _, _, dbg = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, debug=True)
    for b in range(4):
        for s in range(2):
            cand, kept = dbg["cand"][b, s], dbg["kept"][b, s]
            assert len(set(cand.tolist())) == 48 and len(set(kept.tolist())) == 24
            assert set(kept.tolist()) <= set(cand.tolist())
            assert np.all(np.diff(cand) > 0) and np.all(np.diff(kept) > 0)
            # the candidates are the top-48 screening scores
            sc = dbg["score"][b, s]
            assert sc[cand].min() >= np.delete(sc, cand).max()


def test_exact_recovery_never_increases_error(tiny):
    """With exact activations, the recovered term is sum_{i not in K} a_i
    (Ubar V^T)_i = (a_K'^T W) P_V, the projection of the skipped part onto
    the top-r right singular subspace, so the error cannot grow (up to the
    bf16 rounding of the factors)."""
    W, sk, lr = tiny
    x = synth.tokens(256, 8, seed=10)
    _, yd = O.forward_dense(x, W, top_e=2)
    for k in (8, 24, 64):
        _, y_rec, _ = O.forward(x, W, sk, lr, k=k, c=2 * k, r=8, top_e=2, exact_mode=True)
        _, y_no, _ = O.forward(x, W, sk, None, k=k, c=2 * k, r=0, top_e=2, exact_mode=True)
        assert np.linalg.norm(y_rec - yd) <= np.linalg.norm(y_no - yd) * 1.01


def test_combine_identical_experts_gives_that_expert():
    shape = synth.BlockShape(E=4, I=32, d=256, top_e=2)
    W = synth.layer_weights(shape, seed=3)
    for n in ("w_gate", "w_up", "w_down"):
        W[n] = W[n][:1].repeat(4, 1, 1)
    sk = O.build_sketch(W["w_gate"], W["w_up"], 1)
    x = synth.tokens(256, 1, seed=11)
    _, y64, dbg = O.forward(x, W, sk, None, k=8, c=16, r=0, top_e=2, debug=True)
    assert np.allclose(y64[0], dbg["y_expert"][0, 0], rtol=1e-6, atol=1e-9)


# ----------------------------------------------------------------- low rank
def test_lowrank_eckart_young_and_sign_rule():
    W = synth.layer_weights(synth.BlockShape(E=1, I=96, d=256, top_e=1), seed=4)["w_down"][0]
    Wf = O.bf16_to_f64(W)
    r = 8
    ubar, V, S = O.lowrank_f64(W, r)
    resid = np.linalg.norm(Wf - ubar @ V.T) ** 2
    # ||W||_F^2 - sum_{j<=r} sigma_j^2, computed from W and the map itself
    assert np.isclose(resid, np.linalg.norm(Wf) ** 2 - np.linalg.norm(ubar) ** 2, rtol=1e-9)
    assert np.allclose(V.T @ V, np.eye(r), atol=1e-12)
    # best rank r: random rank-r projections do worse
    rng = np.random.default_rng(0)
    for _ in range(5):
        Q, _ = np.linalg.qr(rng.standard_normal((256, r)))
        assert np.linalg.norm(Wf - Wf @ Q @ Q.T) ** 2 > resid
    for p in range(r):
        j = np.argmax(np.abs(V[:, p]))
        assert V[j, p] > 0
    full_u, full_v, _ = O.lowrank_f64(W, 96)
    assert np.allclose(full_u @ full_v.T, Wf, atol=1e-12)


# ------------------------------------------------------------ bf16 rounding
def test_double_to_bf16_matches_torch_rne_on_floats():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(10000).astype(np.float32),
                        np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, 1.0])])
    want = synth.bf16_bits(torch.from_numpy(v).to(torch.bfloat16))
    assert np.array_equal(O.f64_to_bf16(v.astype(np.float64)), want)


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(8)
    x = bf16(rng.standard_normal((2, 256)) * 3)
    h = O.bf16_to_f64(O.rmsnorm(x))
    assert np.allclose(np.sqrt((h ** 2).mean(1)), 1, rtol=1e-2)
    h2 = O.bf16_to_f64(O.rmsnorm(bf16(O.bf16_to_f64(x) * 4)))
    assert np.array_equal(h, h2)


def test_oracle_tiny_forward_regression():
    """The oracle still produces the stored tiny-block outputs."""
    from tests.golden import make_golden
    y, dbg = make_golden.compute()
    rec = {}
    for line in open(os.path.join(GOLDEN, "tiny_forward.txt")):
        if not line.startswith("#"):
            k, *v = line.split()
            rec[k] = v
    assert dbg["ids"].ravel().tolist() == [int(v) for v in rec["ids"]]
    for s in range(2):
        assert dbg["cand"][0, s].tolist() == [int(v) for v in rec[f"cand{s}"]]
        assert dbg["kept"][0, s].tolist() == [int(v) for v in rec[f"kept{s}"]]
    assert y.ravel().tolist() == [int(v, 16) for v in rec["y"]]


def test_openmp_pairs_give_the_same_bits(tiny):
    """The oracle's OpenMP variant runs the (token, slot) readers in
    parallel and combines serially: every output and stage value equals the
    single-threaded run bit for bit, whatever the thread count."""
    W, sk, lr = tiny
    x = synth.tokens(256, 7, seed=21)
    ref = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, debug=True)
    for threads in (2, 5, 16):
        got = O.forward(x, W, sk, lr, k=24, c=48, r=8, top_e=2, debug=True, threads=threads)
        assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1])
        for n in ref[2]:
            assert np.array_equal(ref[2][n], got[2][n]), n
