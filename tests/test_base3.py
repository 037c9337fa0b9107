"""Base-3 sketch packing (five trits per byte) in the oracle: the layout that
brings the resident sketch to the pages' "about 7%" of the BF16 weights
("KAIST: MoE Decoding Needs No Calibration Data", section "A reader that needs
no data at all").  Pinned by hand-derived bytes, an independent decoder and
the round trip through the 2-bit sketch the reader uses."""
import numpy as np
import pytest

from calibration_free_channel_b200 import accounting, synth
from oracle import oracle as O


def _decode(packed, d):
    """Independent decoder: repeated division by 3, digit - 1."""
    out = []
    for b in packed.tolist():
        for _ in range(5):
            out.append(b % 3 - 1)
            b //= 3
    return np.array(out[:d], np.int8)


@pytest.mark.parametrize("trits,byte", [
    ([0, 0, 0, 0, 0], 121),      # digits 1,1,1,1,1: 1 + 3 + 9 + 27 + 81
    ([1, 0, 0, 0, 0], 122),
    ([0, 1, 0, 0, 0], 124),
    ([0, 0, 0, 0, -1], 40),
    ([-1, -1, -1, -1, -1], 0),
    ([1, 1, 1, 1, 1], 242),
])
def test_hand_derived_bytes(trits, byte):
    assert O.pack_trits_base3(np.array(trits, np.int8)).tolist() == [byte]


def test_tail_is_padded_with_zero_trits():
    t = np.array([0, 0, 0, 0, 0, 1, -1], np.int8)
    p = O.pack_trits_base3(t)
    assert p.tolist() == [121, 2 + 0 * 3 + 1 * 9 + 1 * 27 + 1 * 81]


@pytest.mark.parametrize("d", [5, 7, 256, 2048, 2051])
def test_round_trip_and_independent_decoder(d):
    rng = np.random.default_rng(d)
    t = rng.integers(-1, 2, d).astype(np.int8)
    p = O.pack_trits_base3(t)
    assert p.size == (d + 4) // 5 and p.max() <= 242
    assert np.array_equal(O.unpack_trits_base3(p, d), t)
    assert np.array_equal(_decode(p, d), t)


def test_same_trits_as_the_two_bit_sketch():
    W = synth.layer_weights(synth.TINY, seed=0)
    _, skg, _, _, _ = O.build_sketch(W["w_gate"], W["w_up"], synth.rot_seed(0))
    d = 256
    row = skg[3, 17]
    t2 = np.array([O.lib().orc_unpack_trit(O._p(np.ascontiguousarray(row)), j) for j in range(d)], np.int8)
    assert np.array_equal(O.unpack_trits_base3(O.pack_trits_base3(t2), d), t2)


def test_footprints_of_the_qwen3_layer():
    # 2-bit codes: 512-byte rows; base 3: 410 bytes, 416 with whole sectors
    assert accounting.sketch_row_bytes(2048, "2bit") == 512
    assert accounting.sketch_row_bytes(2048, "base3") == 416
    f2 = accounting.sketch_footprint(768, 2048, "2bit")
    f3 = accounting.sketch_footprint(768, 2048, "base3")
    assert abs(f2 - 0.0840) < 1e-4 and abs(f3 - 0.0684) < 1e-4
    assert abs(f3 - 0.07) < abs(f2 - 0.07)  # closer to the pages' about 7%


def test_multiply_shift_divisions_are_exact():
    """The GPU decode of a base-3 byte takes floor(b / 3^k) for k = 1..4 as one
    multiply and shift each on two bytes packed in 16-bit lanes (b * 171 >> 9,
    b * 57 >> 9, b * 19 >> 9, b * 203 >> 14).  For every byte value a packing
    can hold (0..242) they are exact, and no product leaves its 16-bit lane."""
    for b in range(243):
        assert (b * 171) >> 9 == b // 3
        assert (b * 57) >> 9 == b // 9
        assert (b * 19) >> 9 == b // 27
        assert (b * 203) >> 14 == b // 81
        assert max(b * 171, b * 57, b * 19, b * 203) < 1 << 16
        # the digits the decode forms from them are the base-3 digits
        f = [b, (b * 171) >> 9, (b * 57) >> 9, (b * 19) >> 9, (b * 203) >> 14]
        digits = [f[k] - 3 * f[k + 1] for k in range(4)] + [f[4]]
        assert digits == [(b // 3 ** k) % 3 for k in range(5)]
