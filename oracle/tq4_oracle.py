"""CPU oracle for attention over a paged TQ4 KV cache (plain fp64 numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports this module.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may call it. It shares no code, table or constant generator
with the CUDA library; the only thing both consume is the seeded input module.

What it computes, and where each step comes from (JustFit pages):

[BUDGET]  simpleprog.com, "Fitting a 27B-Parameter LLM into 24 GiB of Laptop
          Memory", section "The Memory Budget Equation": 16 full-attention layers,
          4 KV heads of dim 256; a retained position costs 16,640 B over the
          attention layers in four-bit TurboQuant form vs 65,536 B in FP16;
          3,640 MiB vs 14,336 MiB at 229,376 positions.
[KVEXEC]  same page, section "KVExec: Fused Reconstruction with Layer-Scoped
          Lifetime": each vector is 32 U32 words holding eight indices each plus
          one FP16 norm; reconstruction reads the packed page IDs, looks up
          centroids, applies an inverse Hadamard rotation, restores the norm and
          feeds scaled dot-product attention; kernels are specialised to
          256-dim heads and 256-token pages.
[STATE]   same page, section "StateTrans: Request Transitions at Safe
          Boundaries": 256-position pages, shared prefixes by reference count.
[V2]      wpnews.pro, "JustFit: Run Qwen 27B Fast with its full 256K context on
          a 24 GB Mac", mechanism table, row KVExec: rotated-domain attention.

Readings where the pages are silent (each one is a choice, stated here):
 * codebook: 16-level Lloyd-Max quantiser for N(0, 1/256) coordinates, solved and
   used in fp64: encode picks the nearest fp64 centroid (the decision boundaries
   are the midpoints of adjacent centroids) and decode looks the fp64 value up.
   How an implementation stores the table is its own affair; the oracle is the
   definition;
 * rotation: R = H diag(s) / 16 with H the 256x256 Sylvester Hadamard matrix and
   s the seeded +-1 sign diagonal (signs applied first when rotating); the
   inverse is R^T = diag(s) H / 16;
 * norm: ||x||_2 in fp64, stored as fp16 (round to nearest even); the unit
   vector x/||x|| uses the unrounded norm; a zero vector stores norm 0 and
   indices 0;
 * quantiser: nearest centroid, ties to the lower index;
 * packing: coordinate 8w+i is nibble i (bits 4i..4i+3) of word w;
 * page layout (per layer, 266,240 B per 256-position page):
     K words [4 heads][256 slots][32 u32], then V words (same shape),
     then K norms [4][256] fp16, then V norms [4][256] fp16;
   position p of a request lives in page table[p // 256], slot p % 256;
 * GQA: query head h reads KV head h // 6;
 * decode with n_q query tokens over T positions (the n_q new ones included):
   token t attends to positions [0, T - n_q + t];
 * prefill: chunk token i attends to the whole TQ4 prefix and to chunk tokens
   0..i, whose K/V enter attention at their full (bf16) precision.
Parity of the nibble order, the sign-diagonal convention and the page layout is
a convention shared by both sides, not something the pages fix.
"""
from __future__ import annotations

import numpy as np
from scipy.special import ndtr, ndtri

D = 256
PAGE = 256
H_KV = 4
H_Q = 24
GROUP = H_Q // H_KV
WORDS = D // 8
LEVELS = 16

VECTOR_BYTES = WORDS * 4 + 2                 # 130
LAYER_POSITION_BYTES = 2 * H_KV * VECTOR_BYTES  # 1,040
PAGE_BYTES = PAGE * LAYER_POSITION_BYTES       # 266,240
_K_WORDS = 0
_V_WORDS = H_KV * PAGE * WORDS * 4             # 131,072
_K_NORMS = 2 * _V_WORDS                        # 262,144
_V_NORMS = _K_NORMS + H_KV * PAGE * 2          # 264,192


# ----------------------------------------------------------------------------
# codebook [KVEXEC "centroid lookup"; law: Lloyd-Max for N(0, 1/256)]
# ----------------------------------------------------------------------------
def _phi(z):
    return np.exp(-0.5 * z * z) / np.sqrt(2.0 * np.pi)


def lloyd_max_gaussian(levels: int = LEVELS, sigma: float = 1.0 / 16.0,
                       tol: float = 1e-16, max_iter: int = 1_000_000):
    """Lloyd-Max quantiser for N(0, sigma^2): returns (centroids[levels], boundaries[levels-1]).

    Lloyd's two conditions, iterated from equiprobable quantiles until the
    centroids stop moving: each boundary is the midpoint of its two centroids;
    each centroid is the conditional mean E[X | cell], which for a Gaussian is
    sigma * (phi(a) - phi(b)) / (Phi(b) - Phi(a)) on the standardised cell (a, b).
    """
    c = sigma * ndtri((np.arange(levels) + 0.5) / levels)
    for _ in range(max_iter):
        b = 0.5 * (c[:-1] + c[1:])
        lo = np.concatenate(([-np.inf], b)) / sigma
        hi = np.concatenate((b, [np.inf])) / sigma
        mass = ndtr(hi) - ndtr(lo)
        c_new = sigma * (_phi(lo) - _phi(hi)) / mass
        moved = np.max(np.abs(c_new - c))
        c = c_new
        if moved <= tol:
            break
    return c, 0.5 * (c[:-1] + c[1:])


def codebook(levels: int = LEVELS, sigma: float = 1.0 / 16.0):
    """The codebook encode and decode use: the fp64 Lloyd-Max centroids for
    N(0, sigma^2) and, as nearest-centroid decision boundaries, the midpoints of
    adjacent centroids (both float64)."""
    return lloyd_max_gaussian(levels, sigma)


def quantiser_mse(centroids, boundaries, sigma: float = 1.0 / 16.0) -> float:
    """Mean squared error of a scalar quantiser on N(0, sigma^2), summed over its cells.

    For a standardised cell (a, b) with centroid c, the truncated Gaussian
    moments m0 = Phi(b) - Phi(a), m1 = phi(a) - phi(b) and
    m2 = m0 + a phi(a) - b phi(b) give
    int_a^b (sigma z - c)^2 phi(z) dz = sigma^2 m2 - 2 sigma c m1 + c^2 m0.
    """
    lo = np.concatenate(([-np.inf], boundaries)) / sigma
    hi = np.concatenate((boundaries, [np.inf])) / sigma
    m0 = ndtr(hi) - ndtr(lo)
    m1 = _phi(lo) - _phi(hi)
    with np.errstate(invalid="ignore"):   # (+-inf) * 0 at the two open cells; replaced by 0
        lo_t = np.where(np.isfinite(lo), lo * _phi(lo), 0.0)
        hi_t = np.where(np.isfinite(hi), hi * _phi(hi), 0.0)
    m2 = m0 + lo_t - hi_t
    c = np.asarray(centroids)
    return float(np.sum(sigma * sigma * m2 - 2.0 * sigma * c * m1 + c * c * m0))


# ----------------------------------------------------------------------------
# rotation [KVEXEC "inverse Hadamard rotation"; sign diagonal: seeded input]
# ----------------------------------------------------------------------------
def hadamard_matrix(d: int = D) -> np.ndarray:
    """Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j), unnormalised."""
    i = np.arange(d)
    parity = np.bitwise_count(i[:, None] & i[None, :]) & 1
    return np.where(parity == 0, 1.0, -1.0)


def rotation_matrix(signs) -> np.ndarray:
    """R = H diag(s) / sqrt(256): orthogonal; the encoder applies R, decode applies R^T."""
    s = np.asarray(signs, dtype=np.float64)
    return hadamard_matrix(D) * s[None, :] / np.sqrt(D)


# ----------------------------------------------------------------------------
# encode / decode of single vectors [KVEXEC: 32 U32 words + one FP16 norm]
# ----------------------------------------------------------------------------
def nearest_centroid(y, centroids) -> np.ndarray:
    """Index of the nearest centroid for every entry of y; exact ties go to the lower index."""
    y = np.asarray(y, dtype=np.float64)
    dist = np.abs(y[..., None] - np.asarray(centroids)[None, :])
    return np.argmin(dist, axis=-1).astype(np.uint8)  # argmin keeps the first minimum


def pack_indices(idx) -> np.ndarray:
    """[..., 256] indices 0..15 -> [..., 32] uint32, coordinate 8w+i in bits 4i..4i+3 of word w."""
    idx = np.asarray(idx, dtype=np.uint32).reshape(*np.shape(idx)[:-1], WORDS, 8)
    shifts = (4 * np.arange(8, dtype=np.uint32))
    return np.bitwise_or.reduce(idx << shifts, axis=-1).astype(np.uint32)


def unpack_indices(words) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint32)
    shifts = (4 * np.arange(8, dtype=np.uint32))
    idx = (w[..., :, None] >> shifts) & np.uint32(0xF)
    return idx.reshape(*w.shape[:-1], D).astype(np.uint8)


def encode_vectors(x, signs, centroids, block: int = 8192):
    """Quantise head vectors x [..., 256].

    Returns (words [..., 32] uint32, norm16 [...] float16, y [..., 256] float64)
    where y = R x / ||x|| are the rotated unit coordinates the indices quantise
    (returned so that tests can see how close each coordinate is to a boundary).
    Steps: norm -> normalise -> rotate -> nearest centroid -> pack; norm -> fp16.
    Vectors are independent; they are processed ``block`` at a time only to bound memory.
    """
    x = np.asarray(x, dtype=np.float64)
    lead = x.shape[:-1]
    xf = x.reshape(-1, D)
    R = rotation_matrix(signs)
    words = np.empty((xf.shape[0], WORDS), np.uint32)
    norm = np.empty(xf.shape[0], np.float64)
    yall = np.empty_like(xf)
    for a in range(0, xf.shape[0], block):
        xb = xf[a:a + block]
        n = np.sqrt(np.sum(xb * xb, axis=1))
        zero = n == 0.0
        u = xb / np.where(zero, 1.0, n)[:, None]
        y = u @ R.T
        idx = nearest_centroid(y, centroids)
        idx[zero] = 0
        words[a:a + block] = pack_indices(idx)
        norm[a:a + block] = n
        yall[a:a + block] = y
    return (words.reshape(*lead, WORDS), norm.astype(np.float16).reshape(lead),
            yall.reshape(*lead, D))


def decode_vectors(words, norm16, signs, centroids) -> np.ndarray:
    """Reconstruct x_hat = fp16 norm * R^T c[idx] (fp64), the four steps of the KVExec reconstruction."""
    idx = unpack_indices(words)
    c = np.asarray(centroids, dtype=np.float64)[idx]
    R = rotation_matrix(signs)
    unit = c @ R                      # rows: (R^T c)^T = c^T R
    return unit * np.asarray(norm16, dtype=np.float64)[..., None]


# ----------------------------------------------------------------------------
# paged pool [KVEXEC "packed page IDs", 256-token pages; STATE page size 256]
# ----------------------------------------------------------------------------
def new_pool(num_pages: int) -> np.ndarray:
    return np.zeros(num_pages * PAGE_BYTES, np.uint8)


def _regions(pool: np.ndarray):
    pages = pool.reshape(-1, PAGE_BYTES)
    kw = pages[:, _K_WORDS:_V_WORDS].view('<u4').reshape(-1, H_KV, PAGE, WORDS)
    vw = pages[:, _V_WORDS:_K_NORMS].view('<u4').reshape(-1, H_KV, PAGE, WORDS)
    kn = pages[:, _K_NORMS:_V_NORMS].view('<f2').reshape(-1, H_KV, PAGE)
    vn = pages[:, _V_NORMS:PAGE_BYTES].view('<f2').reshape(-1, H_KV, PAGE)
    return kw, vw, kn, vn


def _locate(page_table, positions):
    positions = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(page_table, dtype=np.int64)[positions // PAGE]
    return pages, positions % PAGE


def encode_append(pool, page_table, start_pos, k_new, v_new, signs, centroids):
    """Encode n new positions (K and V [n, 4, 256]) into the pool at [start_pos, start_pos + n).

    Returns the rotated coordinates (yk, yv) for boundary checks.
    """
    k_new = np.asarray(k_new, dtype=np.float64)
    v_new = np.asarray(v_new, dtype=np.float64)
    n = k_new.shape[0]
    kw, vw, kn, vn = _regions(pool)
    pg, slot = _locate(page_table, np.arange(start_pos, start_pos + n))
    wk, nk, yk = encode_vectors(k_new, signs, centroids)
    wv, nv, yv = encode_vectors(v_new, signs, centroids)
    for h in range(H_KV):
        kw[pg, h, slot] = wk[:, h]
        vw[pg, h, slot] = wv[:, h]
        kn[pg, h, slot] = nk[:, h]
        vn[pg, h, slot] = nv[:, h]
    return yk, yv


def gather_packed(pool, page_table, start, n):
    """Packed state of positions [start, start + n): words [n, 4, 32] and norms [n, 4], K then V."""
    kw, vw, kn, vn = _regions(pool)
    pg, slot = _locate(page_table, np.arange(start, start + n))
    out = []
    for arr in (kw, kn, vw, vn):
        out.append(np.stack([arr[pg, h, slot] for h in range(H_KV)], axis=1))
    return out[0], out[1], out[2], out[3]


def reconstruct(pool, page_table, start, n, signs, centroids):
    """Explicit K and V [n, 4, 256] (fp64) for positions [start, start + n) of one request."""
    kw, kn, vw, vn = gather_packed(pool, page_table, start, n)
    return (decode_vectors(kw, kn, signs, centroids),
            decode_vectors(vw, vn, signs, centroids))


# ----------------------------------------------------------------------------
# attention [KVEXEC "immediately consumed by scaled dot-product attention"]
# ----------------------------------------------------------------------------
def sdpa_row(q, K, V, scale):
    """One query row: softmax(scale * K q) V in fp64 (the max is subtracted before exp)."""
    s = scale * (K @ q)
    p = np.exp(s - np.max(s))
    return (p @ V) / np.sum(p)


def decode_attention(pool, page_tables, seq_lens, q, scale, signs, centroids):
    """Decode attention of n_q query tokens per request over its paged TQ4 history.

    q: [n_req, n_q, 24, 256] (bf16 values as floats). seq_lens[r] counts the
    n_q new positions, which must already be in the pool. Token t of request r
    attends to positions [0, seq_lens[r] - n_q + t]. Returns fp64 [n_req, n_q, 24, 256].
    """
    q = np.asarray(q, dtype=np.float64)
    n_req, n_q = q.shape[:2]
    out = np.zeros(q.shape, np.float64)
    for r in range(n_req):
        T = int(seq_lens[r])
        K, V = reconstruct(pool, page_tables[r], 0, T, signs, centroids)
        for t in range(n_q):
            visible = T - n_q + t + 1
            for h in range(H_Q):
                g = h // GROUP
                out[r, t, h] = sdpa_row(q[r, t, h], K[:visible, g], V[:visible, g], scale)
    return out


def prefill_attention(pool, page_table, prefix_len, q, k_chunk, v_chunk, scale, signs,
                      centroids, rows=None):
    """Causal attention of a query chunk against the TQ4 prefix plus the chunk itself.

    q: [n_tok, 24, 256]; k_chunk, v_chunk: [n_tok, 4, 256] at full precision.
    Token i sees prefix positions [0, prefix_len) and chunk tokens 0..i.
    ``rows`` selects which chunk tokens to compute (all by default); the result
    has shape [len(rows), 24, 256].
    """
    q = np.asarray(q, dtype=np.float64)
    n_tok = q.shape[0]
    rows = np.arange(n_tok) if rows is None else np.asarray(rows)
    Kp, Vp = reconstruct(pool, page_table, 0, prefix_len, signs, centroids)
    K = np.concatenate([Kp, np.asarray(k_chunk, dtype=np.float64)], axis=0)
    V = np.concatenate([Vp, np.asarray(v_chunk, dtype=np.float64)], axis=0)
    out = np.zeros((len(rows), H_Q, D), np.float64)
    for j, i in enumerate(rows):
        visible = prefix_len + int(i) + 1
        for h in range(H_Q):
            g = h // GROUP
            out[j, h] = sdpa_row(q[i, h], K[:visible, g], V[:visible, g], scale)
    return out
