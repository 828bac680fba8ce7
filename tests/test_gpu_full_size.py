"""Parity at the workloads' full sizes, in the launch configuration bench.py times.

Decode over 32,768 positions, over 212,992 positions with 5% x8 norms, over two
requests of 163,840 + 65,536 positions (4 causal query tokens each, 64 shared
pages) and over eight one-token requests sharing 32,768 of their 33,792
positions, the last two both ungrouped and grouped (shared pages read once), and
the two-request verify also on the tensor-memory (tcgen05) kernel;
prefill of 2,048 tokens on a 32,768-position prefix, on the packed path and by
direct inverse reconstruction; the prefill's 2,048-token append. For attention the pool is filled with seeded random codes and
norms (every 4-bit value occurs; norms follow the workloads' scale mix), so both
sides read the same bytes and the oracle needs no encoding pass. Decode outputs
are compared in full (fp32 and bf16 outputs); prefill outputs on sampled chunk
tokens, first and last included (the oracle's cost grows with every row)."""
import numpy as np
import pytest

from compressed_paged_kv_tq4_b200 import inputs as I
from oracle import tq4_oracle as O
import _helpers as H

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from compressed_paged_kv_tq4_b200 import tq4  # noqa: E402

SCALE = 1.0 / 16.0


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _random_pool(w, layer=0):
    """A whole pool of random codes and norms (same bytes for the GPU and the oracle)."""
    pool = O.new_pool(w.pool_pages)
    kw, vw, kn, vn = O._regions(pool)
    nw = kw.size
    kw[...] = I.random_codes(w.config, 2 * layer, nw).reshape(kw.shape)
    vw[...] = I.random_codes(w.config, 2 * layer + 1, nw).reshape(vw.shape)
    kn[...] = I.random_norms(w.config, 2 * layer, kn.size, outlier_frac=w.outlier_frac).reshape(kn.shape)
    vn[...] = I.random_norms(w.config, 2 * layer + 1, vn.size, outlier_frac=w.outlier_frac).reshape(vn.shape)
    return pool


@pytest.fixture(scope="module")
def codebook():
    return O.codebook()


@pytest.mark.parametrize("name", ["decode_32k", "decode_213k_outliers", "verify_2req_229k", "shared_prefix_8req_33k"])
def test_decode_full_size(codebook, name):
    c, _ = codebook
    w = I.WORKLOADS[name]
    signs = I.signs(w.config)
    ctx = tq4.Context(signs)
    pool = _random_pool(w)
    tab = I.request_tables(w)
    seq = np.asarray(w.seq_lens, np.int32)
    qb = I.queries(w.config, 0, (w.n_req, w.n_q, 24, 256))
    dpool, dtab, dseq = torch.from_numpy(pool).cuda(), torch.from_numpy(tab).cuda(), torch.from_numpy(seq).cuda()
    q = _bf16_tensor(qb)
    got32 = ctx.decode_attention(dpool, q, dtab, dseq, int(seq.sum()), SCALE, out_dtype=torch.float32)
    got16 = ctx.decode_attention(dpool, q, dtab, dseq, int(seq.sum()), SCALE, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    exp = O.decode_attention(pool, tab, seq, I.bf16_bits_to_f32(qb).astype(np.float64), SCALE, signs, c)
    g32 = got32.cpu().numpy().astype(np.float64)
    assert np.abs(g32 - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), name
    H.assert_bf16_close(got16.float().cpu().numpy(), exp, name)
    if w.n_q > 1:   # the tensor-memory kernel (tcgen05) on the same full-size call
        ctx.set_decode_path(tq4.DECODE_PATH_TENSOR_MEMORY)
        tm32 = ctx.decode_attention(dpool, q, dtab, dseq, int(seq.sum()), SCALE, out_dtype=torch.float32)
        tm16 = ctx.decode_attention(dpool, q, dtab, dseq, int(seq.sum()), SCALE, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        ctx.set_decode_path(tq4.DECODE_PATH_WARP_MMA)
        assert ctx.status() == tq4.TQ4_OK
        t32 = tm32.cpu().numpy().astype(np.float64)
        assert np.abs(t32 - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), name + " tensor memory"
        H.assert_bf16_close(tm16.float().cpu().numpy(), exp, name + " tensor memory")
    if w.shared_prefix_pages:   # the grouped decode: every request led by request 0
        leader, pages = [0] * w.n_req, [w.shared_prefix_pages] * w.n_req
        sh32 = ctx.decode_attention_shared(dpool, q, dtab, dseq, int(seq.sum()), SCALE, leader, pages,
                                           out_dtype=torch.float32)
        sh16 = ctx.decode_attention_shared(dpool, q, dtab, dseq, int(seq.sum()), SCALE, leader, pages,
                                           out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert ctx.status() == tq4.TQ4_OK
        s32 = sh32.cpu().numpy().astype(np.float64)
        assert np.abs(s32 - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), name + " grouped"
        H.assert_bf16_close(sh16.float().cpu().numpy(), exp, name + " grouped")


@pytest.mark.parametrize("reconstruct", [False, True])
def test_prefill_full_size(codebook, reconstruct):
    c, _ = codebook
    w = I.WORKLOADS["prefill_2k_on_32k"]
    signs = I.signs(w.config)
    ctx = tq4.Context(signs)
    pool = _random_pool(w)
    tab = I.request_tables(w)[0]
    qb = I.queries(w.config, 0, (w.n_q, 24, 256))
    kb, vb = I.chunk_kv(w.config, 0, w.n_q)
    out = ctx.prefill_attention(torch.from_numpy(pool).cuda(), torch.from_numpy(tab).cuda(), w.prefix_len,
                                _bf16_tensor(qb), _bf16_tensor(kb), _bf16_tensor(vb), SCALE, reconstruct=reconstruct)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    out32 = ctx.prefill_attention(torch.from_numpy(pool).cuda(), torch.from_numpy(tab).cuda(), w.prefix_len,
                                  _bf16_tensor(qb), _bf16_tensor(kb), _bf16_tensor(vb), SCALE,
                                  out_dtype=torch.float32, reconstruct=reconstruct)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    # 64 chunk tokens: first and last, both sides of every 256-row CTA pair boundary, and a seeded draw
    fixed = np.array([0, 1, 21, 22, 42, 43, 1023, w.n_q - 2, w.n_q - 1])
    others = np.setdiff1d(np.arange(w.n_q), fixed)
    rows = np.sort(np.concatenate([fixed, np.random.default_rng(7).choice(others, 64 - len(fixed), replace=False)]))
    exp = O.prefill_attention(pool, tab, w.prefix_len, I.bf16_bits_to_f32(qb), I.bf16_bits_to_f32(kb),
                              I.bf16_bits_to_f32(vb), SCALE, signs, c, rows=rows)
    H.assert_bf16_close(out.float().cpu().numpy()[rows], exp, "prefill 2048 on 32768")
    err = np.abs(out32.cpu().numpy()[rows].astype(np.float64) - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), err


def test_chunk_append_full_size(codebook):
    """The prefill step's append: 2,048 bf16 tokens at position 32,768 (8 whole pages)."""
    c, b = codebook
    w = I.WORKLOADS["prefill_2k_on_32k"]
    signs = I.signs(w.config)
    ctx = tq4.Context(signs)
    tab = I.request_tables(w)[0]
    kb, vb = I.chunk_kv(w.config, 0, w.n_q)
    pool = tq4.Context.new_pool(w.pool_pages)
    ctx.encode_append(pool, torch.from_numpy(tab).cuda(), w.prefix_len, _bf16_tensor(kb), _bf16_tensor(vb))
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    kf, vf = I.bf16_bits_to_f32(kb), I.bf16_bits_to_f32(vb)
    opool = O.new_pool(w.pool_pages)
    yk, yv = O.encode_append(opool, tab, w.prefix_len, kf, vf, signs, c)
    gkw, gvw, gkn, gvn = O._regions(pool.cpu().numpy())
    okw, ovw, okn, ovn = O._regions(opool)
    pos = np.arange(w.prefix_len, w.prefix_len + w.n_q)
    pg, sl = tab[pos // 256], pos % 256
    nk = H.check_words_against_oracle(gkw[pg, :, sl], okw[pg, :, sl], yk, b, "K words")
    nv = H.check_words_against_oracle(gvw[pg, :, sl], ovw[pg, :, sl], yv, b, "V words")
    H.check_norms_against_oracle(gkn[pg, :, sl], okn[pg, :, sl], kf, "K norms")
    H.check_norms_against_oracle(gvn[pg, :, sl], ovn[pg, :, sl], vf, "V norms")
    assert nk + nv <= 20
