"""CPU oracle for the 2- and 3-bit variants of the paged TurboQuant KV cache (plain fp64 numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports this module.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may call it. It shares no code, table or constant generator
with the CUDA library; it reuses the four-bit oracle's own rotation, quantiser
solver and attention row (oracle/tq4_oracle.py), which are bit-width independent.

The pages describe the four-bit format only ([KVEXEC] simpleprog.com, "Fitting a
27B-Parameter LLM into 24 GiB of Laptop Memory", section "KVExec": 32 U32 words
of eight indices plus one FP16 norm per 256-dim head vector). The scope's
"other bit widths" variant is read here as the same method at b = 2 or 3 bits
per coordinate, every other step unchanged:
 * codebook: the 2^b-level Lloyd-Max quantiser for N(0, 1/256) coordinates,
   solved and used in fp64 (decision boundaries at the midpoints);
 * rotation, norm, nearest-centroid quantiser (ties low), GQA and causal rules:
   exactly those of the four-bit oracle;
 * packing, 8 b u32 words per vector (b = 2: 16 words, b = 3: 24 words):
     plane 0, words 0..15: the low two bits of every index, coordinate 16w + i in
       bits 2i..2i+1 of word w;
     plane 1 (b = 3 only), words 16..23: bit 2 of every index, coordinate
       32w + i in bit i of word 16 + w;
 * page layout (per layer, 256 positions): K words [4 heads][256 slots][8 b u32],
   then V words (same shape), then K norms [4][256] fp16, then V norms; a layer-
   position is 8 x (32 b + 2) B: 528 B (b = 2), 784 B (b = 3).
"""
from __future__ import annotations

import numpy as np

from oracle import tq4_oracle as T4

D = T4.D
PAGE = T4.PAGE
H_KV = T4.H_KV
H_Q = T4.H_Q
GROUP = T4.GROUP
BITS = (2, 3)


def words_per_vector(bits: int) -> int:
    return 8 * bits


def vector_bytes(bits: int) -> int:
    return 4 * words_per_vector(bits) + 2


def layer_position_bytes(bits: int) -> int:
    return 2 * H_KV * vector_bytes(bits)


def page_bytes(bits: int) -> int:
    return PAGE * layer_position_bytes(bits)


def _offsets(bits: int):
    wb = H_KV * PAGE * words_per_vector(bits) * 4
    kn = 2 * wb
    vn = kn + H_KV * PAGE * 2
    return 0, wb, kn, vn, page_bytes(bits)


def codebook(bits: int, sigma: float = 1.0 / 16.0):
    """The 2^bits-level fp64 Lloyd-Max centroids for N(0, sigma^2) and their midpoint boundaries."""
    assert bits in BITS
    return T4.lloyd_max_gaussian(1 << bits, sigma)


# ----------------------------------------------------------------------------
# packing (the bit-plane reading above)
# ----------------------------------------------------------------------------
def pack_indices(idx, bits: int) -> np.ndarray:
    """[..., 256] indices 0..2^bits - 1 -> [..., 8 bits] uint32."""
    idx = np.asarray(idx, dtype=np.uint32)
    lead = idx.shape[:-1]
    lo = (idx & np.uint32(3)).reshape(*lead, 16, 16)
    plane0 = np.bitwise_or.reduce(lo << (2 * np.arange(16, dtype=np.uint32)), axis=-1).astype(np.uint32)
    if bits == 2:
        return plane0
    hi = ((idx >> np.uint32(2)) & np.uint32(1)).reshape(*lead, 8, 32)
    plane1 = np.bitwise_or.reduce(hi << np.arange(32, dtype=np.uint32), axis=-1).astype(np.uint32)
    return np.concatenate([plane0, plane1], axis=-1)


def unpack_indices(words, bits: int) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint32)
    lead = w.shape[:-1]
    lo = (w[..., :16, None] >> (2 * np.arange(16, dtype=np.uint32))) & np.uint32(3)
    idx = lo.reshape(*lead, D)
    if bits == 3:
        hi = (w[..., 16:24, None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
        idx = idx | (hi.reshape(*lead, D) << np.uint32(2))
    return idx.astype(np.uint8)


# ----------------------------------------------------------------------------
# encode / decode of single vectors
# ----------------------------------------------------------------------------
def encode_vectors(x, signs, centroids, bits: int):
    """Quantise head vectors x [..., 256]: returns (words [..., 8 bits] uint32,
    norm16 [...] float16, y [..., 256] the rotated unit coordinates).
    Steps, as for four bits: norm -> normalise -> rotate -> nearest centroid -> pack."""
    x = np.asarray(x, dtype=np.float64)
    lead = x.shape[:-1]
    xf = x.reshape(-1, D)
    n = np.sqrt(np.sum(xf * xf, axis=1))
    zero = n == 0.0
    u = xf / np.where(zero, 1.0, n)[:, None]
    y = u @ T4.rotation_matrix(signs).T
    idx = T4.nearest_centroid(y, centroids)
    idx[zero] = 0
    words = pack_indices(idx, bits)
    return (words.reshape(*lead, words_per_vector(bits)), n.astype(np.float16).reshape(lead),
            y.reshape(*lead, D))


def decode_vectors(words, norm16, signs, centroids, bits: int) -> np.ndarray:
    """x_hat = fp16 norm * R^T c[idx] (fp64)."""
    c = np.asarray(centroids, dtype=np.float64)[unpack_indices(words, bits)]
    return (c @ T4.rotation_matrix(signs)) * np.asarray(norm16, dtype=np.float64)[..., None]


# ----------------------------------------------------------------------------
# paged pool
# ----------------------------------------------------------------------------
def new_pool(num_pages: int, bits: int) -> np.ndarray:
    return np.zeros(num_pages * page_bytes(bits), np.uint8)


def _regions(pool: np.ndarray, bits: int):
    k0, v0, kn0, vn0, pb = _offsets(bits)
    wv = words_per_vector(bits)
    pages = pool.reshape(-1, pb)
    kw = pages[:, k0:v0].view('<u4').reshape(-1, H_KV, PAGE, wv)
    vw = pages[:, v0:kn0].view('<u4').reshape(-1, H_KV, PAGE, wv)
    kn = pages[:, kn0:vn0].view('<f2').reshape(-1, H_KV, PAGE)
    vn = pages[:, vn0:pb].view('<f2').reshape(-1, H_KV, PAGE)
    return kw, vw, kn, vn


def encode_append(pool, page_table, start_pos, k_new, v_new, signs, centroids, bits: int):
    """Encode n new positions (K and V [n, 4, 256]) into the pool at [start_pos, start_pos + n)."""
    k_new = np.asarray(k_new, dtype=np.float64)
    v_new = np.asarray(v_new, dtype=np.float64)
    n = k_new.shape[0]
    kw, vw, kn, vn = _regions(pool, bits)
    pos = np.arange(start_pos, start_pos + n)
    pg = np.asarray(page_table, dtype=np.int64)[pos // PAGE]
    slot = pos % PAGE
    wk, nk, yk = encode_vectors(k_new, signs, centroids, bits)
    wvv, nv, yv = encode_vectors(v_new, signs, centroids, bits)
    for h in range(H_KV):
        kw[pg, h, slot] = wk[:, h]
        vw[pg, h, slot] = wvv[:, h]
        kn[pg, h, slot] = nk[:, h]
        vn[pg, h, slot] = nv[:, h]
    return yk, yv


def reconstruct(pool, page_table, start, n, signs, centroids, bits: int):
    """Explicit K and V [n, 4, 256] (fp64) for positions [start, start + n) of one request."""
    kw, vw, kn, vn = _regions(pool, bits)
    pos = np.arange(start, start + n)
    pg = np.asarray(page_table, dtype=np.int64)[pos // PAGE]
    slot = pos % PAGE
    K = np.stack([decode_vectors(kw[pg, h, slot], kn[pg, h, slot], signs, centroids, bits) for h in range(H_KV)], 1)
    V = np.stack([decode_vectors(vw[pg, h, slot], vn[pg, h, slot], signs, centroids, bits) for h in range(H_KV)], 1)
    return K, V


def decode_attention(pool, page_tables, seq_lens, q, scale, signs, centroids, bits: int):
    """Decode attention of n_q query tokens per request over its paged b-bit history
    (the four-bit oracle's rule: token t of a request of length T sees [0, T - n_q + t])."""
    q = np.asarray(q, dtype=np.float64)
    n_req, n_q = q.shape[:2]
    out = np.zeros(q.shape, np.float64)
    for r in range(n_req):
        T = int(seq_lens[r])
        K, V = reconstruct(pool, page_tables[r], 0, T, signs, centroids, bits)
        for t in range(n_q):
            visible = T - n_q + t + 1
            for h in range(H_Q):
                g = h // GROUP
                out[r, t, h] = T4.sdpa_row(q[r, t, h], K[:visible, g], V[:visible, g], scale)
    return out


def prefill_attention(pool, page_table, prefix_len, q, k_chunk, v_chunk, scale, signs, centroids, bits: int,
                      rows=None):
    """Causal attention of a query chunk against the b-bit prefix plus the chunk itself
    (the four-bit oracle's rule: token i sees prefix positions [0, prefix_len) and chunk
    tokens 0..i; the chunk's K/V at full precision). ``rows`` selects chunk tokens."""
    q = np.asarray(q, dtype=np.float64)
    n_tok = q.shape[0]
    rows = np.arange(n_tok) if rows is None else np.asarray(rows)
    Kp, Vp = reconstruct(pool, page_table, 0, prefix_len, signs, centroids, bits)
    K = np.concatenate([Kp, np.asarray(k_chunk, dtype=np.float64)], axis=0)
    V = np.concatenate([Vp, np.asarray(v_chunk, dtype=np.float64)], axis=0)
    out = np.zeros((len(rows), H_Q, D), np.float64)
    for j, i in enumerate(rows):
        visible = prefix_len + int(i) + 1
        for h in range(H_Q):
            g = h // GROUP
            out[j, h] = T4.sdpa_row(q[i, h], K[:visible, g], V[:visible, g], scale)
    return out
