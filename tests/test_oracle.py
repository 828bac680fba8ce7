"""Pins for the CPU oracle: it is checked against what the pages print, against
textbook values, closed forms and invariants, never against itself.

Runs without a GPU.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import tq4_oracle as O
from compressed_paged_kv_tq4_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MIB = 1 << 20


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def solution():
    """The fp64 Lloyd-Max solution (pinned against Max 1960)."""
    return O.lloyd_max_gaussian()


@pytest.fixture(scope="module")
def codebook():
    """The codebook that encode/decode use (fp64 centroids, midpoint boundaries)."""
    return O.codebook()


@pytest.fixture(scope="module")
def signs():
    return I.signs(0)


# --------------------------------------------------------------------------- bytes
def test_byte_accounting_matches_pages():
    g = _golden("pages_byte_accounting.json")
    layers = g["attention_layers"]["value"]
    heads = g["kv_heads"]["value"]
    d = g["head_dim"]["value"]
    assert O.D == d and O.H_KV == heads and O.PAGE == g["page_positions"]["value"]
    assert O.WORDS == g["words_per_vector"]["value"]
    assert d // O.WORDS == g["indices_per_word"]["value"]
    # one vector: 32 u32 + one fp16 norm
    assert O.VECTOR_BYTES == 4 * g["words_per_vector"]["value"] + 2 == 130
    per_pos = layers * O.LAYER_POSITION_BYTES
    assert per_pos == g["tq4_bytes_per_position_all_layers"]["value"]
    fp16_per_pos = layers * heads * 2 * d * 2
    assert fp16_per_pos == g["fp16_bytes_per_position_all_layers"]["value"]
    n = g["pool_positions"]["value"]
    assert n * per_pos / MIB == g["tq4_mib_at_pool"]["value"]
    assert n * fp16_per_pos / MIB == g["fp16_mib_at_pool"]["value"]
    assert round(fp16_per_pos / per_pos, g["reduction_printed"]["digits"]) == g["reduction_printed"]["value"]
    b = g["bf16_one_layer_192k_mib"]
    assert b["positions"] * heads * 2 * d * 2 / MIB == b["value"]
    h = g["lm_head_mib"]
    assert round(h["value"] * MIB / per_pos) == h["equivalent_positions"]
    # the oracle's page holds exactly 256 layer-positions
    assert O.new_pool(1).nbytes == O.PAGE_BYTES == O.PAGE * O.LAYER_POSITION_BYTES


def test_gathered_state_is_1040_bytes_per_position(codebook, signs):
    pool = O.new_pool(2)
    rng = np.random.default_rng(3)
    k, v = rng.standard_normal((2, 5, 4, 256))
    O.encode_append(pool, [1, 0], 250, k, v, signs, codebook[0])
    kw, kn, vw, vn = O.gather_packed(pool, [1, 0], 250, 5)
    per_pos = (kw.nbytes + kn.nbytes + vw.nbytes + vn.nbytes) // 5
    assert per_pos == 1040


# --------------------------------------------------------------------------- codebook
def test_codebook_matches_max_1960(solution):
    g = _golden("lloyd_max_gaussian_16.json")
    c, b = solution
    unit_c = c * 16.0
    unit_b = b * 16.0
    def unit_in_last_place(v):
        return 10.0 ** (math.floor(math.log10(abs(v))) - g["significant_figures"] + 1) if v else 1e-4

    for got, printed in zip(unit_c[8:], g["output_levels"]):
        assert abs(got - printed) <= unit_in_last_place(printed)
    for got, printed in zip(unit_b[7:], g["transition_points"]):
        assert abs(got - printed) <= unit_in_last_place(printed)
    mse = O.quantiser_mse(unit_c, unit_b, sigma=1.0)
    assert abs(mse - g["mean_squared_error"]) < 1e-5


def test_codebook_symmetric_and_midpoints(solution):
    c, b = solution
    assert np.all(np.diff(c) > 0)
    assert np.max(np.abs(c + c[::-1])) < 1e-15
    assert np.allclose(b, 0.5 * (c[1:] + c[:-1]), atol=0, rtol=0)


def test_codebook_used_is_the_fp64_solution(solution, codebook):
    """Encode and decode use the fp64 Lloyd-Max centroids themselves (no rounding
    of the table) and the midpoints of adjacent centroids as boundaries."""
    c, b = solution
    cu, bu = codebook
    assert cu.dtype == np.float64 and bu.dtype == np.float64
    assert np.array_equal(cu, c) and np.array_equal(bu, b)
    # a table rounded to fp16 (or bf16) is a different table: it fails this pin
    assert not np.array_equal(cu, c.astype(np.float16).astype(np.float64))
    assert np.max(np.abs(cu - c.astype(np.float16).astype(np.float64))) > 1e-5


def test_codebook_centroids_are_monte_carlo_conditional_means(solution):
    c, b = solution
    x = np.random.default_rng(11).standard_normal(20_000_000) / 16.0
    cell = np.searchsorted(b, x)
    sums = np.bincount(cell, weights=x, minlength=16)
    counts = np.bincount(cell, minlength=16)
    mc = sums / counts
    # standard error of the outermost cell mean is ~5e-5 in these units
    assert np.max(np.abs(mc - c)) < 3e-4
    mse = np.mean((x - c[cell]) ** 2) * 256.0
    assert abs(mse - O.quantiser_mse(c * 16, b * 16, 1.0)) < 2e-5


# --------------------------------------------------------------------------- rotation
def test_hadamard_is_sylvester_and_orthogonal():
    H = O.hadamard_matrix(256)
    assert np.array_equal(H @ H, 256.0 * np.eye(256))
    assert np.array_equal(H, H.T)
    # built independently by the doubling recursion [[H, H], [H, -H]]
    S = np.array([[1.0]])
    while S.shape[0] < 256:
        S = np.block([[S, S], [S, -S]])
    assert np.array_equal(H, S)


def test_hadamard_equals_butterflies():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 256))
    y = x.copy()
    h = 1
    while h < 256:  # in-place radix-2 butterflies
        y = y.reshape(7, -1, 2, h)
        a, b = y[:, :, 0, :].copy(), y[:, :, 1, :].copy()
        y[:, :, 0, :], y[:, :, 1, :] = a + b, a - b
        y = y.reshape(7, 256)
        h *= 2
    assert np.allclose(y, x @ O.hadamard_matrix(256).T, atol=1e-12, rtol=0)


def test_rotation_orthogonal_signs_first(signs):
    R = O.rotation_matrix(signs)
    assert np.allclose(R @ R.T, np.eye(256), atol=1e-14)
    # applying R to a basis vector e_i: sign i first, then column i of H / 16
    H = O.hadamard_matrix(256)
    for i in (0, 1, 77, 255):
        e = np.zeros(256)
        e[i] = 1.0
        assert np.array_equal(R @ e, signs[i] * H[:, i] / 16.0)


# --------------------------------------------------------------------------- packing / quantiser
def test_pack_nibble_order_hand_computed():
    idx = np.arange(256) % 16
    words = O.pack_indices(idx)
    assert words.dtype == np.uint32 and words.shape == (32,)
    assert all(int(w) == (0x76543210 if i % 2 == 0 else 0xFEDCBA98) for i, w in enumerate(words))
    rng = np.random.default_rng(2)
    r = rng.integers(0, 16, (9, 256))
    assert np.array_equal(O.unpack_indices(O.pack_indices(r)), r)


def test_quantiser_ties_go_lower(codebook):
    # exact ties need exactly representable distances: a dyadic codebook
    toy = np.array([-1.5, -0.5, 0.5, 1.5])
    assert O.nearest_centroid(np.array([-1.0, 0.0, 1.0, 7.0, -7.0]), toy).tolist() == [0, 1, 2, 3, 0]
    c, b = codebook
    assert np.array_equal(O.nearest_centroid(b - 1e-12, c), np.arange(15))
    assert np.array_equal(O.nearest_centroid(b + 1e-12, c), np.arange(1, 16))
    assert np.array_equal(O.nearest_centroid(c, c), np.arange(16))
    assert O.nearest_centroid(np.array([-1.0, 1.0]), c).tolist() == [0, 15]


def test_encode_decode_relative_mse_within_codebook_bound(codebook, signs):
    c, b = codebook
    rng = np.random.default_rng(7)
    x = rng.standard_normal((20000, 256)) * rng.uniform(0.5, 2.0, (20000, 1))
    w, n, _ = O.encode_vectors(x, signs, c)
    xh = O.decode_vectors(w, n, signs, c)
    rel = np.sum((x - xh) ** 2, axis=1) / np.sum(x * x, axis=1)
    bound = O.quantiser_mse(c, b)  # distortion per coordinate of a unit vector x 256 coordinates
    assert abs(np.mean(rel) / (bound * 256) - 1.0) < 0.10


def test_norm_is_fp16_of_l2_norm(codebook, signs):
    rng = np.random.default_rng(8)
    x = rng.standard_normal((50, 256)) * 3
    _, n, _ = O.encode_vectors(x, signs, codebook[0])
    assert n.dtype == np.float16
    assert np.array_equal(n, np.linalg.norm(x, axis=1).astype(np.float16))


def test_zero_vector_encodes_to_zero(codebook, signs):
    w, n, _ = O.encode_vectors(np.zeros((1, 256)), signs, codebook[0])
    assert not w.any() and float(n[0]) == 0.0
    assert not O.decode_vectors(w, n, signs, codebook[0]).any()


def test_reconstruction_points_are_fixed_points(codebook, signs):
    """Re-encoding a reconstruction gives the same words, and the norm of the
    reconstruction (norm * ||c[idx]||) rounded to fp16. Index vectors come from
    encoding Gaussian data, so ||c[idx]|| is within ~1% of 1 and every rescaled
    centroid stays inside its own cell."""
    c, _ = codebook
    rng = np.random.default_rng(9)
    words, _, _ = O.encode_vectors(rng.standard_normal((64, 256)), signs, c)
    idx = O.unpack_indices(words)
    norm = rng.uniform(1, 40, 64).astype(np.float16)
    xh = O.decode_vectors(words, norm, signs, c)
    w2, n2, _ = O.encode_vectors(xh, signs, c)
    assert np.array_equal(w2, words)
    expect = (norm.astype(np.float64) * np.linalg.norm(c[idx], axis=1)).astype(np.float16)
    assert np.array_equal(n2, expect)


def test_rotated_domain_identity(codebook, signs):
    """q . x_hat = n * (R q) . c[idx]: scores can be taken in the rotated domain."""
    c, _ = codebook
    rng = np.random.default_rng(10)
    x = rng.standard_normal((30, 256))
    q = rng.standard_normal(256)
    w, n, _ = O.encode_vectors(x, signs, c)
    xh = O.decode_vectors(w, n, signs, c)
    R = O.rotation_matrix(signs)
    rot = n.astype(np.float64) * (c[O.unpack_indices(w)] @ (R @ q))
    assert np.allclose(xh @ q, rot, atol=1e-12, rtol=1e-12)


# --------------------------------------------------------------------------- pool
def test_pool_byte_layout(codebook, signs):
    c, _ = codebook
    pool = O.new_pool(3)
    table = [2, 0, 1]
    rng = np.random.default_rng(12)
    k, v = rng.standard_normal((2, 1, 4, 256))
    pos = 300  # page-table entry 1 -> physical page 0, slot 44
    O.encode_append(pool, table, pos, k, v, signs, c)
    wk, nk, _ = O.encode_vectors(k[0], signs, c)
    wv, nv, _ = O.encode_vectors(v[0], signs, c)
    base = 0 * O.PAGE_BYTES
    for h in range(4):
        off = base + (h * 256 + 44) * 128
        assert pool[off:off + 128].tobytes() == wk[h].astype("<u4").tobytes()
        off = base + 131072 + (h * 256 + 44) * 128
        assert pool[off:off + 128].tobytes() == wv[h].astype("<u4").tobytes()
        off = base + 262144 + (h * 256 + 44) * 2
        assert pool[off:off + 2].tobytes() == nk[h:h + 1].astype("<f2").tobytes()
        off = base + 264192 + (h * 256 + 44) * 2
        assert pool[off:off + 2].tobytes() == nv[h:h + 1].astype("<f2").tobytes()
    touched = np.flatnonzero(pool)
    assert touched.min() >= 0 and touched.max() < O.PAGE_BYTES  # only physical page 0


# --------------------------------------------------------------------------- attention
def _pool_with(k, v, table, signs, c):
    pool = O.new_pool(max(table) + 1)
    O.encode_append(pool, table, 0, k, v, signs, c)
    return pool


def test_single_key_returns_reconstructed_value(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(13)
    k, v = rng.standard_normal((2, 1, 4, 256))
    pool = _pool_with(k, v, [0], signs, c)
    q = rng.standard_normal((1, 1, 24, 256))
    out = O.decode_attention(pool, [[0]], [1], q, 1 / 16, signs, c)
    _, vh = O.reconstruct(pool, [0], 0, 1, signs, c)
    for h in range(24):
        assert np.allclose(out[0, 0, h], vh[0, h // 6], atol=1e-13)


def test_gqa_head_mapping(codebook, signs):
    """With one key, query head h returns V of KV head h // 6; the four V heads differ."""
    c, _ = codebook
    rng = np.random.default_rng(14)
    k = rng.standard_normal((1, 4, 256))
    v = np.stack([np.full(256, float(g + 1)) * (1 + 0.5 * np.arange(256) / 256) for g in range(4)])[None]
    pool = _pool_with(k, v, [0], signs, c)
    out = O.decode_attention(pool, [[0]], [1], rng.standard_normal((1, 1, 24, 256)), 1 / 16, signs, c)
    _, vh = O.reconstruct(pool, [0], 0, 1, signs, c)
    means = [vh[0, g].mean() for g in range(4)]
    assert len(set(np.round(means, 6))) == 4
    for h in range(24):
        assert np.allclose(out[0, 0, h], vh[0, h // 6], atol=1e-12)


def test_zero_query_gives_mean_value(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(15)
    k, v = rng.standard_normal((2, 37, 4, 256))
    pool = _pool_with(k, v, [0], signs, c)
    out = O.decode_attention(pool, [[0]], [37], np.zeros((1, 1, 24, 256)), 1 / 16, signs, c)
    _, vh = O.reconstruct(pool, [0], 0, 37, signs, c)
    for h in range(24):
        assert np.allclose(out[0, 0, h], vh[:, h // 6].mean(axis=0), atol=1e-13)


def test_two_keys_logistic_closed_form(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(16)
    k, v = rng.standard_normal((2, 2, 4, 256))
    pool = _pool_with(k, v, [0], signs, c)
    q = rng.standard_normal((1, 1, 24, 256))
    scale = 0.37
    out = O.decode_attention(pool, [[0]], [2], q, scale, signs, c)
    kh, vh = O.reconstruct(pool, [0], 0, 2, signs, c)
    for h in range(24):
        g = h // 6
        delta = scale * (q[0, 0, h] @ kh[0, g] - q[0, 0, h] @ kh[1, g])
        w0 = 1.0 / (1.0 + math.exp(-delta))
        assert np.allclose(out[0, 0, h], w0 * vh[0, g] + (1 - w0) * vh[1, g], atol=1e-12)


def test_causal_tokens_match_shorter_single_token_decode(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(17)
    T = 300
    k, v = rng.standard_normal((2, T, 4, 256))
    table = [1, 0]
    pool = _pool_with(k, v, table, signs, c)
    q = rng.standard_normal((1, 4, 24, 256))
    out4 = O.decode_attention(pool, [table], [T], q, 1 / 16, signs, c)
    for t in range(4):
        out1 = O.decode_attention(pool, [table], [T - 4 + t + 1], q[:, t:t + 1], 1 / 16, signs, c)
        assert np.allclose(out4[0, t], out1[0, 0], atol=1e-13)


def test_page_table_permutation_invariance(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(18)
    T = 700
    k, v = rng.standard_normal((2, T, 4, 256))
    q = rng.standard_normal((1, 1, 24, 256))
    outs = []
    for table in ([0, 1, 2], [2, 0, 1], [1, 2, 0]):
        pool = _pool_with(k, v, table, signs, c)
        outs.append(O.decode_attention(pool, [table], [T], q, 1 / 16, signs, c))
    assert np.allclose(outs[0], outs[1], atol=0, rtol=0)
    assert np.allclose(outs[0], outs[2], atol=0, rtol=0)


def _fixed_point_vectors(rng, n, signs, c):
    """Vectors that decode(encode(x)) returns unchanged: x = m R^T c[idx] with
    ||c[idx]|| within 1e-5 of 1 (so the fp16 norm of x is m exactly)."""
    R = O.rotation_matrix(signs)
    out = np.empty((n, 256))
    for i in range(n):
        idx = rng.integers(0, 16, 256)
        for _ in range(20000):
            s2 = np.sum(c[idx] ** 2)
            if abs(math.sqrt(s2) - 1.0) < 1e-5:
                break
            j = rng.integers(256)
            step = -1 if s2 > 1.0 else 1
            if c[idx[j]] < 0:
                step = -step
            idx[j] = min(15, max(0, idx[j] + step))
        assert abs(math.sqrt(np.sum(c[idx] ** 2)) - 1.0) < 1e-5
        m = float(np.float16(rng.uniform(2, 30)))
        out[i] = m * (c[idx] @ R)
    return out


def test_fixed_point_attention_equals_full_precision(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(19)
    T = 20
    kv = _fixed_point_vectors(rng, 2 * T * 4, signs, c).reshape(2, T, 4, 256)
    k, v = kv
    pool = _pool_with(k, v, [0], signs, c)
    kh, vh = O.reconstruct(pool, [0], 0, T, signs, c)
    assert np.allclose(kh, k, atol=1e-12) and np.allclose(vh, v, atol=1e-12)
    q = rng.standard_normal((1, 1, 24, 256))
    out = O.decode_attention(pool, [[0]], [T], q, 1 / 16, signs, c)
    for h in range(24):  # plain softmax written as a logistic-free normalised sum
        s = np.array([np.dot(q[0, 0, h], k[j, h // 6]) / 16 for j in range(T)])
        w = np.exp(s) / np.exp(s).sum()
        assert np.allclose(out[0, 0, h], w @ v[:, h // 6], atol=1e-12)


def test_prefill_matches_decode_on_fixed_point_chunk(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(20)
    P, n = 270, 6
    kp, vp = rng.standard_normal((2, P, 4, 256))
    kc, vc = _fixed_point_vectors(rng, 2 * n * 4, signs, c).reshape(2, n, 4, 256)
    table = [1, 0]
    pool = O.new_pool(2)
    O.encode_append(pool, table, 0, kp, vp, signs, c)
    q = rng.standard_normal((n, 24, 256))
    pre = O.prefill_attention(pool, table, P, q, kc, vc, 1 / 16, signs, c)
    O.encode_append(pool, table, P, kc, vc, signs, c)
    for i in range(n):
        dec = O.decode_attention(pool, [table], [P + i + 1], q[None, i:i + 1], 1 / 16, signs, c)
        assert np.allclose(pre[i], dec[0, 0], atol=1e-12)


def test_prefill_first_token_without_prefix_returns_its_value(codebook, signs):
    c, _ = codebook
    rng = np.random.default_rng(21)
    q = rng.standard_normal((3, 24, 256))
    kc, vc = rng.standard_normal((2, 3, 4, 256))
    pre = O.prefill_attention(O.new_pool(1), [0], 0, q, kc, vc, 1 / 16, signs, c)
    for h in range(24):
        assert np.allclose(pre[0, h], vc[0, h // 6], atol=1e-14)


def test_tq4_attention_close_to_full_precision(codebook, signs):
    """Brute force on a tiny input: TQ4 attention is within the codebook error of fp attention."""
    c, _ = codebook
    rng = np.random.default_rng(22)
    T = 3
    k, v = rng.standard_normal((2, T, 4, 256))
    pool = _pool_with(k, v, [0], signs, c)
    q = rng.standard_normal((1, 1, 24, 256))
    out = O.decode_attention(pool, [[0]], [T], q, 1 / 16, signs, c)
    for h in range(24):
        s = np.array([q[0, 0, h] @ k[j, h // 6] / 16 for j in range(T)])
        w = np.exp(s - s.max())
        full = (w / w.sum()) @ v[:, h // 6]
        # relative reconstruction error ~ sqrt(0.0095) ~ 0.1 of |v| per key
        assert np.max(np.abs(out[0, 0, h] - full)) < 0.5
