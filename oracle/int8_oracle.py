"""CPU oracle for the uniform INT8 comparison arm (plain fp64 numpy).

TEST INFRASTRUCTURE ONLY, like tq4_oracle.py: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` may call it, and it shares no code
with the CUDA library.

What it computes. The JustFit page (simpleprog.com, "Fitting a 27B-Parameter
LLM into 24 GiB of Laptop Memory", section "Reasoning at 200K") runs the same
long-context workload with "a uniform INT8 comparison" arm next to TQ4 and says
nothing more about it. Readings taken here (each a choice):
 * uniform, symmetric quantisation of each 256-dim K or V head vector on its own:
   scale s = max_i |x_i| / 127 (fp64), codes q_i = round-half-to-even(x_i / s),
   which lie in [-127, 127]; the scale is stored as fp16 (round to nearest even)
   and the codes with the unrounded scale, as the TQ4 norm is; a zero vector
   stores scale 0 and codes 0;
 * no rotation and no codebook: reconstruction is x_hat = fp16(s) * q;
 * storage per layer-position: 4 heads x (K + V) x (256 int8 + one fp16) = 2,064 B;
   page layout (256 positions): K codes [4][256][256] int8, V codes (same shape),
   K scales [4][256] fp16, V scales [4][256] fp16: 528,384 B per page;
 * attention exactly as for TQ4 (GQA 24 / 4, softmax in fp64 here), over the
   reconstructed K/V; decode token t of n_q sees [0, T - n_q + t].
"""
from __future__ import annotations

import numpy as np

from oracle import tq4_oracle as T4

D = 256
PAGE = 256
H_KV = 4
H_Q = 24
GROUP = H_Q // H_KV

VECTOR_BYTES = D + 2                               # 258
LAYER_POSITION_BYTES = 2 * H_KV * VECTOR_BYTES     # 2,064
PAGE_BYTES = PAGE * LAYER_POSITION_BYTES            # 528,384
_K_CODES = 0
_V_CODES = H_KV * PAGE * D                         # 262,144
_K_SCALES = 2 * _V_CODES                           # 524,288
_V_SCALES = _K_SCALES + H_KV * PAGE * 2            # 526,336


def encode_vectors(x):
    """x [..., 256] -> (codes int8 [..., 256], scale16 float16 [...], ratio float64 [..., 256]).

    ratio = x / s (the value each code rounds), returned so that tests can see how
    close a coordinate is to a rounding midpoint."""
    x = np.asarray(x, dtype=np.float64)
    s = np.max(np.abs(x), axis=-1) / 127.0
    zero = s == 0.0
    ratio = x / np.where(zero, 1.0, s)[..., None]
    q = np.rint(ratio)                                  # numpy rounds half to even
    q[zero] = 0.0
    return q.astype(np.int8), s.astype(np.float16), ratio


def decode_vectors(codes, scale16):
    """x_hat = fp16 scale * codes (fp64)."""
    return np.asarray(codes, np.float64) * np.asarray(scale16, np.float64)[..., None]


def new_pool(num_pages: int) -> np.ndarray:
    return np.zeros(num_pages * PAGE_BYTES, np.uint8)


def _regions(pool):
    pages = pool.reshape(-1, PAGE_BYTES)
    kc = pages[:, _K_CODES:_V_CODES].view(np.int8).reshape(-1, H_KV, PAGE, D)
    vc = pages[:, _V_CODES:_K_SCALES].view(np.int8).reshape(-1, H_KV, PAGE, D)
    ks = pages[:, _K_SCALES:_V_SCALES].view('<f2').reshape(-1, H_KV, PAGE)
    vs = pages[:, _V_SCALES:PAGE_BYTES].view('<f2').reshape(-1, H_KV, PAGE)
    return kc, vc, ks, vs


def encode_append(pool, page_table, start_pos, k_new, v_new):
    """Encode n new positions (K, V [n, 4, 256]) at [start_pos, start_pos + n).
    Returns the ratios (K, V) for rounding-midpoint checks."""
    n = np.asarray(k_new).shape[0]
    kc, vc, ks, vs = _regions(pool)
    pos = np.arange(start_pos, start_pos + n)
    pg, slot = np.asarray(page_table, np.int64)[pos // PAGE], pos % PAGE
    qk, sk, rk = encode_vectors(k_new)
    qv, sv, rv = encode_vectors(v_new)
    for h in range(H_KV):
        kc[pg, h, slot] = qk[:, h]
        vc[pg, h, slot] = qv[:, h]
        ks[pg, h, slot] = sk[:, h]
        vs[pg, h, slot] = sv[:, h]
    return rk, rv


def reconstruct(pool, page_table, start, n):
    """Explicit K and V [n, 4, 256] (fp64) for positions [start, start + n)."""
    kc, vc, ks, vs = _regions(pool)
    pos = np.arange(start, start + n)
    pg, slot = np.asarray(page_table, np.int64)[pos // PAGE], pos % PAGE
    K = np.stack([decode_vectors(kc[pg, h, slot], ks[pg, h, slot]) for h in range(H_KV)], axis=1)
    V = np.stack([decode_vectors(vc[pg, h, slot], vs[pg, h, slot]) for h in range(H_KV)], axis=1)
    return K, V


def decode_attention(pool, page_tables, seq_lens, q, scale):
    """As tq4_oracle.decode_attention, over the INT8 cache. q [n_req, n_q, 24, 256]."""
    q = np.asarray(q, dtype=np.float64)
    n_req, n_q = q.shape[:2]
    out = np.zeros(q.shape, np.float64)
    for r in range(n_req):
        T = int(seq_lens[r])
        K, V = reconstruct(pool, page_tables[r], 0, T)
        for t in range(n_q):
            visible = T - n_q + t + 1
            for h in range(H_Q):
                g = h // GROUP
                out[r, t, h] = T4.sdpa_row(q[r, t, h], K[:visible, g], V[:visible, g], scale)
    return out
