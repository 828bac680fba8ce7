"""Pins of the 2- and 3-bit oracle (oracle/tqb_oracle.py) against things it does
not compute itself: Max's published Lloyd-Max tables for 4 and 8 levels
(tests/golden/), byte counts derived by hand from the packing reading, packed
words built bit by bit, brute-force nearest centroids, exact reconstruction of
vectors whose rotated coordinates are centroids, and attention closed forms."""
import json
import math
import os

import numpy as np
import pytest

from compressed_paged_kv_tq4_b200 import inputs as I
from oracle import tqb_oracle as OB
from oracle import tq4_oracle as O4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("bits,fixture", [(2, "lloyd_max_gaussian_4.json"), (3, "lloyd_max_gaussian_8.json")])
def test_codebook_matches_max_1960(bits, fixture):
    g = _golden(fixture)
    c, b = OB.codebook(bits)
    levels = 1 << bits
    unit_c, unit_b = c * 16.0, b * 16.0

    def ulp(v):
        return 10.0 ** (math.floor(math.log10(abs(v))) - g["significant_figures"] + 1) if v else 1e-4

    for got, printed in zip(unit_c[levels // 2:], g["output_levels"]):
        assert abs(got - printed) <= ulp(printed), (got, printed)
    for got, printed in zip(unit_b[levels // 2 - 1:], g["transition_points"]):
        assert abs(got - printed) <= ulp(printed), (got, printed)
    mse = O4.quantiser_mse(unit_c, unit_b, sigma=1.0)
    assert abs(mse - g["mean_squared_error"]) <= g["mse_printed_precision"]


def test_codebook_symmetric_midpoints_and_ordering():
    mses = []
    for bits in (2, 3):
        c, b = OB.codebook(bits)
        assert len(c) == 1 << bits and np.all(np.diff(c) > 0)
        assert np.max(np.abs(c + c[::-1])) < 1e-15
        assert np.array_equal(b, 0.5 * (c[1:] + c[:-1]))
        mses.append(O4.quantiser_mse(c, b))
    mses.append(O4.quantiser_mse(*O4.codebook()))
    assert mses[0] > mses[1] > mses[2]          # more levels, less distortion


def test_byte_accounting():
    # 256 coordinates x b bits / 8 + one fp16 norm, 8 vectors (4 heads x K, V) per layer-position
    assert OB.vector_bytes(2) == 66 and OB.vector_bytes(3) == 98
    assert OB.layer_position_bytes(2) == 528 and OB.layer_position_bytes(3) == 784
    assert OB.page_bytes(2) == 135_168 and OB.page_bytes(3) == 200_704
    for bits in (2, 3):
        pool = OB.new_pool(2, bits)
        kw, vw, kn, vn = OB._regions(pool, bits)
        assert (kw.nbytes + vw.nbytes + kn.nbytes + vn.nbytes) == pool.nbytes


def test_packing_bit_by_bit():
    idx = np.zeros(256, np.uint8)
    idx[17] = 3                       # 2-bit: coordinate 17 = 16*1 + 1 -> bits 2..3 of word 1
    w = OB.pack_indices(idx, 2)
    assert w.shape == (16,) and w[1] == 0b1100 and np.count_nonzero(w) == 1
    idx[:] = 0
    idx[33] = 5                       # 3-bit 0b101: low bits 01 -> word 2 bits 2..3; bit 2 -> word 16 + 1, bit 1
    w = OB.pack_indices(idx, 3)
    assert w.shape == (24,) and w[2] == 0b0100 and w[17] == 0b10 and np.count_nonzero(w) == 2
    idx[:] = 7
    w = OB.pack_indices(idx, 3)
    assert np.all(w[:16] == 0xFFFFFFFF) and np.all(w[16:] == 0xFFFFFFFF)
    rng = np.random.default_rng(3)
    for bits in (2, 3):
        r = rng.integers(0, 1 << bits, size=(5, 256), dtype=np.uint8)
        assert np.array_equal(OB.unpack_indices(OB.pack_indices(r, bits), bits), r)


@pytest.mark.parametrize("bits", [2, 3])
def test_encode_picks_the_nearest_centroid(bits):
    c, _ = OB.codebook(bits)
    signs = I.signs(0)
    x = np.random.default_rng(5).standard_normal((64, 256))
    words, norm16, y = OB.encode_vectors(x, signs, c, bits)
    idx = OB.unpack_indices(words, bits)
    brute = np.array([[int(np.argmin([abs(v - cc) for cc in c])) for v in row] for row in y])
    assert np.array_equal(idx, brute)
    assert np.array_equal(norm16, np.linalg.norm(x, axis=1).astype(np.float16))


@pytest.mark.parametrize("bits", [2, 3])
def test_centroid_vectors_reconstruct_exactly(bits):
    """For the index pattern of a typical unit vector, x = R^T c[idx] has rotated unit
    coordinates c[idx] / |x|, close enough to the centroids (|x| is about 0.94 for
    2 bits, 0.98 for 3) to keep every index; its reconstruction is then exactly
    fp16(|x|) * x."""
    c, _ = OB.codebook(bits)
    signs = I.signs(1)
    g = np.random.default_rng(7).standard_normal((4, 256))
    idx = O4.nearest_centroid(g / np.linalg.norm(g, axis=1, keepdims=True), c)   # a typical index pattern
    x = c[idx] @ O4.rotation_matrix(signs)          # rows: (R^T c[idx])^T
    words, norm16, _ = OB.encode_vectors(x, signs, c, bits)
    assert np.array_equal(OB.unpack_indices(words, bits), idx)
    xh = OB.decode_vectors(words, norm16, signs, c, bits)
    assert np.max(np.abs(xh - x * norm16.astype(np.float64)[:, None])) < 1e-12


@pytest.mark.parametrize("bits", [2, 3])
def test_attention_closed_forms(bits):
    c, _ = OB.codebook(bits)
    signs = I.signs(2)
    rng = np.random.default_rng(9)
    table = np.array([1, 0], np.int32)
    pool = OB.new_pool(2, bits)
    k = rng.standard_normal((3, 4, 256))
    v = rng.standard_normal((3, 4, 256))
    k[1] = k[0]                        # positions 0 and 1: identical keys
    OB.encode_append(pool, table, 0, k, v, signs, c, bits)
    K, V = OB.reconstruct(pool, table, 0, 3, signs, c, bits)
    q = rng.standard_normal((1, 2, 24, 256))
    # one position visible (length 2, two query tokens: token 0 sees position 0 only)
    out = OB.decode_attention(pool, table[None], [2], q, 1 / 16, signs, c, bits)
    for h in range(24):
        assert np.allclose(out[0, 0, h], V[0, h // 6], rtol=0, atol=1e-12)
        # token 1 sees positions 0 and 1, whose keys are equal: the mean of their values
        assert np.allclose(out[0, 1, h], 0.5 * (V[0, h // 6] + V[1, h // 6]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("bits", OB.BITS)
def test_prefill_without_prefix_is_bit_width_independent(bits):
    """With no prefix the chunk attends to itself at full precision, so the b-bit
    prefill must equal the four-bit oracle's prefill of the same chunk."""
    c, _ = OB.codebook(bits)
    c4, _ = O4.codebook()
    signs = I.signs(3)
    rng = np.random.default_rng(11)
    n_tok = 5
    q = rng.standard_normal((n_tok, 24, 256))
    kc = rng.standard_normal((n_tok, 4, 256))
    vc = rng.standard_normal((n_tok, 4, 256))
    got = OB.prefill_attention(OB.new_pool(1, bits), np.zeros(1, np.int32), 0, q, kc, vc, 1 / 16, signs, c, bits)
    exp = O4.prefill_attention(O4.new_pool(1), np.zeros(1, np.int32), 0, q, kc, vc, 1 / 16, signs, c4)
    assert np.array_equal(got, exp)


@pytest.mark.parametrize("bits", OB.BITS)
def test_prefill_zero_query_is_the_mean_of_visible_values(bits):
    """q = 0 makes every visible score equal: token i's output is the plain mean of the
    rebuilt prefix values and the chunk values of tokens 0..i (a wrong window, a
    missing prefix or a wrong page fails it)."""
    c, _ = OB.codebook(bits)
    signs = I.signs(4)
    rng = np.random.default_rng(12)
    table = np.array([2, 0, 1], np.int32)
    pool = OB.new_pool(3, bits)
    prefix = 600
    k = rng.standard_normal((prefix, 4, 256))
    v = rng.standard_normal((prefix, 4, 256)) * rng.uniform(0.5, 2.0, (prefix, 1, 1))
    OB.encode_append(pool, table, 0, k, v, signs, c, bits)
    _, Vp = OB.reconstruct(pool, table, 0, prefix, signs, c, bits)
    n_tok = 4
    kc = rng.standard_normal((n_tok, 4, 256))
    vc = rng.standard_normal((n_tok, 4, 256))
    out = OB.prefill_attention(pool, table, prefix, np.zeros((n_tok, 24, 256)), kc, vc, 1 / 16, signs, c, bits)
    for i in range(n_tok):
        mean = (Vp.sum(axis=0) + vc[:i + 1].sum(axis=0)) / (prefix + i + 1)   # [4, 256]
        for h in range(24):
            assert np.allclose(out[i, h], mean[h // 6], rtol=0, atol=1e-12)
