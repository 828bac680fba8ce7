"""Pins for the uniform INT8 comparison arm's oracle (oracle/int8_oracle.py):
byte accounting, exact round trips, the rounding rule, the quantisation error
bound and closed forms of attention. Runs without a GPU."""
import numpy as np

from oracle import int8_oracle as O8
from oracle import tq4_oracle as O4


def test_byte_accounting():
    # one vector: 256 int8 codes + one fp16 scale; 4 KV heads x (K + V) per layer-position
    assert O8.VECTOR_BYTES == 258
    assert O8.LAYER_POSITION_BYTES == 2 * 4 * 258 == 2064
    assert O8.new_pool(1).nbytes == O8.PAGE_BYTES == 256 * 2064
    # over the 16 attention layers: half of FP16 plus the scales, about twice TQ4
    fp16 = 16 * 4 * 2 * 256 * 2
    assert 16 * O8.LAYER_POSITION_BYTES == fp16 // 2 + 16 * 4 * 2 * 2
    assert 16 * O8.LAYER_POSITION_BYTES / (16 * O4.LAYER_POSITION_BYTES) == 2064 / 1040


def test_fp16_exact_vectors_round_trip_exactly():
    rng = np.random.default_rng(1)
    q = rng.integers(-127, 128, size=(50, 256))
    q[:, 7] = np.where(rng.random(50) < 0.5, 127, -127)        # the absmax element
    s = np.float16(rng.uniform(1e-3, 0.5, 50)).astype(np.float64)
    x = q * s[:, None]
    codes, s16, _ = O8.encode_vectors(x)
    assert np.array_equal(codes.astype(np.int64), q)
    assert np.array_equal(s16.astype(np.float64), s)
    assert np.array_equal(O8.decode_vectors(codes, s16), x)


def test_rounding_is_half_to_even_and_absmax_maps_to_127():
    x = np.zeros(256)
    x[0] = 127.0
    x[1:7] = [2.5, 3.5, -2.5, -3.5, 0.5, 126.5]
    codes, s16, _ = O8.encode_vectors(x)
    assert float(s16) == 1.0
    assert codes[0] == 127 and list(codes[1:7]) == [2, 4, -2, -4, 0, 126]
    codes, _, _ = O8.encode_vectors(-x)
    assert codes[0] == -127


def test_zero_vector():
    codes, s16, _ = O8.encode_vectors(np.zeros((2, 256)))
    assert not codes.any() and not s16.astype(np.float64).any()
    assert not O8.decode_vectors(codes, s16).any()


def test_quantisation_error_bound():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2000, 256)) * rng.uniform(0.5, 16, (2000, 1))
    codes, s16, _ = O8.encode_vectors(x)
    s = np.max(np.abs(x), axis=1) / 127.0
    err = np.abs(O8.decode_vectors(codes, s16) - x)
    bound = s[:, None] / 2 + np.abs(codes) * np.abs(s - s16.astype(np.float64))[:, None]
    assert np.all(err <= bound * (1 + 1e-12))
    assert np.all(np.abs(codes).max(axis=1) == 127)


def test_pool_round_trip_and_attention_closed_forms():
    rng = np.random.default_rng(3)
    pool = O8.new_pool(2)
    table = np.array([1, 0])
    k, v = rng.standard_normal((2, 300, 4, 256))
    O8.encode_append(pool, table, 0, k, v)
    K, V = O8.reconstruct(pool, table, 0, 300)
    codes, s16, _ = O8.encode_vectors(v[299])
    assert np.array_equal(V[299], O8.decode_vectors(codes, s16))
    q = rng.standard_normal((1, 1, 24, 256))
    # one visible position: the output is that position's reconstructed V
    out = O8.decode_attention(pool, table[None], [1], q, 0.0625)
    for h in range(24):
        assert np.allclose(out[0, 0, h], V[0, h // 6], rtol=0, atol=1e-12)
    # zero query: the mean of the visible reconstructed values
    out = O8.decode_attention(pool, table[None], [300], np.zeros((1, 1, 24, 256)), 0.0625)
    assert np.allclose(out[0, 0, 7], V[:, 1].mean(axis=0), rtol=0, atol=1e-12)
    # a brute-force softmax over the reconstructed K/V, written out here
    s = 0.0625 * K[:, 2] @ q[0, 0, 13]
    p = np.exp(s - s.max())
    exp = (p / p.sum()) @ V[:, 2]
    out = O8.decode_attention(pool, table[None], [300], q, 0.0625)
    assert np.allclose(out[0, 0, 13], exp, rtol=0, atol=1e-12)
