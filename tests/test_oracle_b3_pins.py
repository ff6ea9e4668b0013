"""Pins for the oracle's base-3 storage of ternary codes (five codes per byte,
1.6 bits per weight; the pages put the information content of a ternary
weight at log2(3) ~ 1.58 bits: inferownia.pl, "BitNet b1.58: era 1-bitowych
LLM-ów", "Skąd te 1,58 bita"; Habr repost on juhe.plus, "Когда - три лучше
двух").  Tied to hand-worked bytes under tests/golden/, round trips, the
byte range and the 2-bit product on the same codes."""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, vals = line.split(":", 1)
            out[key.strip()] = vals.split()
    return out


def test_b3_layout_fixture(orc):
    gold = _golden("pack_b3_layout_k80.txt")
    K = int(gold["a_K"][0])
    q = np.zeros((1, K), dtype=np.int8)
    for kv in gold["a_nonzero"]:
        k, v = kv.split(":")
        q[0, int(k)] = int(v)
    expect = np.array([[int(b) for b in gold["a_bytes"]]], dtype=np.uint8)
    np.testing.assert_array_equal(orc.pack_codes_b3(q), expect)
    back, bad = orc.unpack_codes_b3(expect, K)
    assert bad == 0
    np.testing.assert_array_equal(back, q)
    # all +1 / all -1 rows
    np.testing.assert_array_equal(orc.pack_codes_b3(np.ones((1, 80), np.int8)), np.full((1, 16), 242, np.uint8))
    np.testing.assert_array_equal(orc.pack_codes_b3(-np.ones((1, 80), np.int8)), np.zeros((1, 16), np.uint8))
    # padded row
    Kc = int(gold["c_K"][0])
    expect_c = np.array([[int(b) for b in gold["c_bytes"]]], dtype=np.uint8)
    np.testing.assert_array_equal(orc.pack_codes_b3(np.ones((1, Kc), np.int8)), expect_c)


@pytest.mark.parametrize("K", [64, 80, 192, 2560, 6912])
def test_b3_roundtrip_size_and_range(orc, K):
    rng = np.random.default_rng(K)
    q = rng.integers(-1, 2, size=(7, K)).astype(np.int8)
    packed = orc.pack_codes_b3(q)
    Kp = (K + 79) // 80 * 80
    assert orc.b3_padded_k(K) == Kp
    assert packed.shape == (7, Kp // 5)
    assert packed.max() <= 242
    back, bad = orc.unpack_codes_b3(packed, K)
    assert bad == 0
    np.testing.assert_array_equal(back, q)
    # 1.6 bits per weight of the padded row: 20% fewer bytes than the 2-bit layout
    assert packed.shape[1] * 8 == Kp * 8 // 5
    if K % 80 == 0:
        assert packed.shape[1] * 5 == orc.pack_codes(q).shape[1] * 4


def test_b3_bytes_are_base3_numbers_of_strided_codes(orc):
    # independent decode with numpy: byte i of group g, digit t <-> weight 80g + 16t + i
    rng = np.random.default_rng(11)
    K = 240
    q = rng.integers(-1, 2, size=(3, K)).astype(np.int8)
    packed = orc.pack_codes_b3(q).astype(np.int64)
    digits = np.stack([(packed // 3 ** t) % 3 for t in range(5)], axis=-1)  # N x bytes x 5
    g = np.arange(packed.shape[1]) // 16
    i = np.arange(packed.shape[1]) % 16
    k = 80 * g[:, None] + 16 * np.arange(5)[None, :] + i[:, None]
    np.testing.assert_array_equal(digits - 1, q[:, k])


def test_b3_invalid_bytes_and_padding_are_counted(orc):
    packed = np.full((1, 16), 121, np.uint8)
    packed[0, 3] = 243
    packed[0, 7] = 255
    _, bad = orc.unpack_codes_b3(packed, 80)
    assert bad == 2
    # K = 64: digit 4 of every byte is padding and must be code 1 (q = 0)
    packed = np.full((1, 16), 121, np.uint8)
    packed[0, 5] = 121 + 81  # padding digit = 2
    _, bad = orc.unpack_codes_b3(packed, 64)
    assert bad == 1


def test_b3_product_equals_2bit_product(orc):
    from bitlinear_absmean_ternary_b200 import synth
    W = synth.weights(40, 6912, 0.02, 0, 7)
    x = synth.activations(3, 6912, 0, 8, "normal", 0.01, 20.0, "bf16")
    p2, g2 = orc.pack_weights(W, 1e-5)
    p3, g3 = orc.pack_weights_b3(W, 1e-5)
    assert g2 == g3
    xq, a, _ = orc.quant_act(x)
    acc2, y2 = orc.bitlinear(p2, g2, 6912, xq, a)
    acc3, y3 = orc.bitlinear_b3(p3, g3, 6912, xq, a)
    np.testing.assert_array_equal(acc3, acc2)
    np.testing.assert_array_equal(y3, y2)
