"""Seeded synthetic inputs for the TQ4 paged-KV attention path.

This module only draws random numbers and shapes them into workloads. It holds
none of the method's arithmetic (no rotation, codebook, quantisation, packing or
attention). Both the CUDA path and the CPU oracle consume what it returns.

Randomness: numpy PCG64 streams keyed by ``SeedSequence([20260915 + config,
purpose, layer])`` so that any single layer of any workload can be regenerated
on its own (the oracle samples layers; the GPU path builds all of them).

Workload shapes follow the JustFit pages (simpleprog.com "Fitting a
27B-Parameter LLM into 24 GiB of Laptop Memory", sections "The Memory Budget
Equation" and "Results"): 16 full-attention layers, 4 KV heads of dim 256,
256-position pages, contexts of 32K, 196,608 + 16,384 and 2 x 112K positions in
a 229,376-position pool. The query side uses 24 heads (GQA group of 6).
"""
from __future__ import annotations

import dataclasses

import numpy as np

SEED_BASE = 20260915

D = 256
PAGE = 256
H_KV = 4
H_Q = 24
POOL_PAGES = 229_376 // PAGE  # 896 pages

# purposes (second SeedSequence word)
_SIGNS, _KV, _OUTLIER, _Q, _TABLE, _NEWKV, _CHUNK, _CODES, _NORMS = range(9)


def _rng(config: int, purpose: int, layer: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([SEED_BASE + int(config), int(purpose), int(layer)])
    return np.random.Generator(np.random.PCG64(ss))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even) and return the raw uint16 bits.

    This defines what a "bf16 input" is for every workload; both sides read
    the same bits. NaN/Inf are not produced by the generators below.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def signs(config: int) -> np.ndarray:
    """The seeded +-1 sign diagonal of the rotation, int8 [256]."""
    r = _rng(config, _SIGNS)
    return (r.integers(0, 2, size=D, dtype=np.int8) * 2 - 1).astype(np.int8)


def kv_vectors(config: int, layer: int, n_pos: int, *, outlier_frac: float = 0.0,
               outlier_scale: float = 8.0, first_pos: int = 0, request: int = 0):
    """K and V head vectors, fp32 [n_pos, 4, 256] each.

    Each vector is z * s with z ~ N(0, I_256) and s ~ U(0.5, 2) drawn per vector.
    With ``outlier_frac`` > 0, a seeded fraction of positions has s multiplied
    by ``outlier_scale`` for all of its K and V vectors.

    Positions are generated page by page (256 positions per draw) so that a
    window [first_pos, first_pos + n_pos) is reproducible on its own. ``request``
    selects an independent stream (two requests that do not share pages).
    """
    k = np.empty((n_pos, H_KV, D), np.float32)
    v = np.empty((n_pos, H_KV, D), np.float32)
    if n_pos == 0:
        return k, v
    p0 = first_pos // PAGE
    p1 = (first_pos + n_pos + PAGE - 1) // PAGE
    for pg in range(p0, p1):
        r = _rng(config, _KV + 16 * request, layer * 1_000_003 + pg)
        z = r.standard_normal((PAGE, 2, H_KV, D), dtype=np.float32)
        s = r.uniform(0.5, 2.0, size=(PAGE, 2, H_KV, 1)).astype(np.float32)
        if outlier_frac > 0.0:
            ro = _rng(config, _OUTLIER + 16 * request, layer * 1_000_003 + pg)
            mask = ro.random(PAGE) < outlier_frac
            s[mask] *= np.float32(outlier_scale)
        blk = z * s
        lo = max(first_pos, pg * PAGE)
        hi = min(first_pos + n_pos, (pg + 1) * PAGE)
        a, b = lo - pg * PAGE, hi - pg * PAGE
        k[lo - first_pos:hi - first_pos] = blk[a:b, 0]
        v[lo - first_pos:hi - first_pos] = blk[a:b, 1]
    return k, v


def kv_vectors_device(config: int, layer: int, n_pos: int, *, outlier_frac: float = 0.0,
                      outlier_scale: float = 8.0, request: int = 0, device="cuda"):
    """K and V head vectors with the distribution of ``kv_vectors``, drawn on the
    GPU with torch's generator: fp32 tensors [n_pos, 4, 256] each.

    Each vector is z * s with z ~ N(0, I_256) and s ~ U(0.5, 2); a seeded
    ``outlier_frac`` of positions has s multiplied by ``outlier_scale`` for all of
    its K and V vectors. The stream differs from ``kv_vectors`` (same law, other
    numbers); it fills the benchmark's multi-GB caches, where only the law
    matters. Parity tests use ``kv_vectors``.
    """
    import torch
    seed = int(np.random.SeedSequence([SEED_BASE + int(config), _KV + 16 * int(request), int(layer)])
               .generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1))
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    k = torch.randn((n_pos, H_KV, D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((n_pos, H_KV, D), generator=g, device=device, dtype=torch.float32)
    sk = torch.rand((n_pos, H_KV, 1), generator=g, device=device) * 1.5 + 0.5
    sv = torch.rand((n_pos, H_KV, 1), generator=g, device=device) * 1.5 + 0.5
    if outlier_frac > 0.0:
        mask = (torch.rand((n_pos, 1, 1), generator=g, device=device) < outlier_frac).float()
        boost = 1.0 + (outlier_scale - 1.0) * mask
        sk = sk * boost
        sv = sv * boost
    return k * sk, v * sv


def queries(config: int, layer: int, shape) -> np.ndarray:
    """N(0,1) queries rounded to bf16; returns uint16 bits of the given shape."""
    r = _rng(config, _Q, layer)
    return to_bf16_bits(r.standard_normal(shape, dtype=np.float32))


def chunk_kv(config: int, layer: int, n_tok: int):
    """N(0,1) K/V for a prefill chunk, bf16 bits [n_tok, 4, 256] each."""
    r = _rng(config, _CHUNK, layer)
    k = r.standard_normal((n_tok, H_KV, D), dtype=np.float32)
    v = r.standard_normal((n_tok, H_KV, D), dtype=np.float32)
    return to_bf16_bits(k), to_bf16_bits(v)


def random_codes(config: int, layer: int, n_words: int) -> np.ndarray:
    """n_words uniformly random uint32 words: every 4-bit field is uniform over 0..15."""
    r = _rng(config, _CODES, layer)
    return r.integers(0, 2 ** 32, size=n_words, dtype=np.uint64).astype(np.uint32)


def random_norms(config: int, layer: int, n: int, *, outlier_frac: float = 0.0,
                 outlier_scale: float = 8.0) -> np.ndarray:
    """n positive fp32 magnitudes 16 s, s ~ U(0.5, 2) (the length of a 256-dim
    N(0, s^2 I) vector is about 16 s); a seeded ``outlier_frac`` of them times
    ``outlier_scale``. The scale mix of ``kv_vectors``, without the vectors."""
    r = _rng(config, _NORMS, layer)
    s = r.uniform(0.5, 2.0, size=n)
    if outlier_frac > 0.0:
        s[r.random(n) < outlier_frac] *= outlier_scale
    return (16.0 * s).astype(np.float32)


def page_table_scattered(config: int, n_pages: int, pool_pages: int = POOL_PAGES,
                         salt: int = 0) -> np.ndarray:
    """n_pages distinct physical page ids drawn from a pool, int32, seeded order."""
    if n_pages > pool_pages:
        raise ValueError("table larger than pool")
    r = _rng(config, _TABLE, salt)
    return r.permutation(pool_pages)[:n_pages].astype(np.int32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One workload: shapes only. Values come from the generators above."""
    name: str
    config: int
    layers: int
    pool_pages: int
    seq_lens: tuple          # attended positions per request (new positions included)
    n_q: int                 # query tokens per request (decode) or chunk length (prefill)
    kind: str                # "decode", "decode_int8" (the INT8 comparison arm), "decode_tqb2" /
                             # "decode_tqb3" (the 2- and 3-bit variants) or "prefill"
    outlier_frac: float = 0.0
    append_per_step: int = 0  # positions appended by tq4_encode_append per layer per step
    shared_prefix_pages: int = 0
    grouped: bool = False    # attend through the shared-prefix (grouped) decode
    prefix_len: int = 0      # prefill only

    @property
    def n_req(self) -> int:
        return len(self.seq_lens)


WORKLOADS = {
    # 1 layer, 1 request, 1 query token, 2,048 positions in 8 pages (table = permutation of 8)
    "single_layer_2k": Workload("single_layer_2k", 0, 1, 8, (2048,), 1, "decode"),
    # 16 layers, 1 request, 1 query token, 32,768 positions scattered in an 896-page pool
    "decode_32k": Workload("decode_32k", 1, 16, POOL_PAGES, (32768,), 1, "decode",
                           append_per_step=1),
    # 16 layers, 212,992 positions (196,608 + 16,384), 5% x8 outliers, append 1 per layer
    "decode_213k_outliers": Workload("decode_213k_outliers", 2, 16, POOL_PAGES, (212_992,), 1,
                                     "decode", outlier_frac=0.05, append_per_step=1),
    # 2 requests (163,840 and 65,536 positions; first 64 pages shared), 4 causal query tokens each
    "verify_2req_229k": Workload("verify_2req_229k", 3, 16, POOL_PAGES, (163_840, 65_536), 4,
                                 "decode", shared_prefix_pages=64, append_per_step=4),
    # 8 requests sharing a 32,768-position prefix (128 pages), 1,024 own positions each,
    # one query token: the grouped decode reads the shared pages once for all eight
    "shared_prefix_8req_33k": Workload("shared_prefix_8req_33k", 5, 16, POOL_PAGES, (33_792,) * 8, 1, "decode",
                                       shared_prefix_pages=128, grouped=True, append_per_step=1),
    # the uniform INT8 comparison arm on the decode_32k shape (same config, same law of K/V)
    "int8_decode_32k": Workload("int8_decode_32k", 1, 16, POOL_PAGES, (32768,), 1, "decode_int8",
                                append_per_step=1),
    # the 3- and 2-bit variants on the decode_32k shape (same config, same law of K/V)
    "tqb3_decode_32k": Workload("tqb3_decode_32k", 1, 16, POOL_PAGES, (32768,), 1, "decode_tqb3",
                                append_per_step=1),
    "tqb2_decode_32k": Workload("tqb2_decode_32k", 1, 16, POOL_PAGES, (32768,), 1, "decode_tqb2",
                                append_per_step=1),
    # prefill: 2,048 causal query tokens against a 32,768-position TQ4 prefix + the chunk
    "prefill_2k_on_32k": Workload("prefill_2k_on_32k", 4, 16, POOL_PAGES, (32_768 + 2048,), 2048,
                                  "prefill", prefix_len=32_768, append_per_step=2048),
}


def request_tables(w: Workload) -> np.ndarray:
    """Page tables [n_req, max_pages] int32 for a workload (unused entries = -1).

    Single request: a seeded draw of distinct pages from the pool (for the 8-page
    pool: a permutation of all 8). Two requests: request 0 gets its pages; request 1
    reuses request 0's first ``shared_prefix_pages`` entries and then fresh pages.
    """
    npg = [(s + PAGE - 1) // PAGE for s in w.seq_lens]
    max_pages = max(npg)
    tab = np.full((w.n_req, max_pages), -1, np.int32)
    if w.n_req == 1:
        tab[0, :npg[0]] = page_table_scattered(w.config, npg[0], w.pool_pages)
        return tab
    total = npg[0] + sum(n - w.shared_prefix_pages for n in npg[1:])
    ids = page_table_scattered(w.config, total, w.pool_pages)
    tab[0, :npg[0]] = ids[:npg[0]]
    off = npg[0]
    for r in range(1, w.n_req):
        tab[r, :w.shared_prefix_pages] = tab[0, :w.shared_prefix_pages]
        fresh = npg[r] - w.shared_prefix_pages
        tab[r, w.shared_prefix_pages:npg[r]] = ids[off:off + fresh]
        off += fresh
    return tab
