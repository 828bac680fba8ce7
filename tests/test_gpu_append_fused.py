"""tq4_decode_append_attention: the step's append and its decode in one call.

It must leave the pool byte-identical to tq4_encode_append of each request's new
positions and return exactly what tq4_decode_attention returns afterwards
(n_q = 1: the encode runs inside the decode kernel; n_q > 1: a tail-encode
kernel). Cases put the new position at both edges of a page and make the last
split short; one case is also checked against the oracle."""
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


def _setup(config, seq_lens, n_q, dtype):
    signs = I.signs(config)
    ctx = tq4.Context(signs)
    npg = [(s + 255) // 256 for s in seq_lens]
    pool_pages = sum(npg) + 3
    ids = I.page_table_scattered(config, sum(npg), pool_pages)
    tab = np.full((len(seq_lens), max(npg)), -1, np.int32)
    off = 0
    for r, n in enumerate(npg):
        tab[r, :n] = ids[off:off + n]
        off += n
    tabs = torch.from_numpy(tab).cuda()
    pool = tq4.Context.new_pool(pool_pages)
    hist, new = [], []
    for r, s in enumerate(seq_lens):
        k, v = I.kv_vectors(config, 0, s, request=r, outlier_frac=0.05)
        if dtype == torch.bfloat16:
            k, v = I.bf16_bits_to_f32(I.to_bf16_bits(k)), I.bf16_bits_to_f32(I.to_bf16_bits(v))
        hist.append((k, v))
        ctx.encode_append(pool, tabs[r], 0, torch.from_numpy(k[:s - n_q]).cuda(),
                          torch.from_numpy(v[:s - n_q]).cuda())
        new.append((k[s - n_q:], v[s - n_q:]))
    k_new = torch.from_numpy(np.stack([a for a, _ in new])).to(device="cuda", dtype=dtype)
    v_new = torch.from_numpy(np.stack([b for _, b in new])).to(device="cuda", dtype=dtype)
    qb = I.queries(config, 0, (len(seq_lens), n_q, 24, 256))
    q = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).cuda()
    seq = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    return ctx, signs, pool, tab, tabs, k_new, v_new, q, qb, seq, hist


@pytest.mark.parametrize("n_q,seq_lens,dtype", [
    (1, [2049], torch.float32),           # new position in slot 0 of a page
    (1, [4096], torch.bfloat16),          # new position in slot 255
    (1, [700, 1300], torch.float32),      # two requests
    (1, [33], torch.bfloat16),            # one short split
    (1, [20000], torch.float32),          # last split: a partial round of 32-position tiles
    (1, [32556], torch.bfloat16),         # last split: a full round, then 16-position tiles
    (2, [1500, 257], torch.float32),
    (4, [2048, 333], torch.bfloat16),
])
def test_fused_append_equals_append_then_decode(n_q, seq_lens, dtype):
    ctx, signs, pool, tab, tabs, k_new, v_new, q, qb, seq, hist = _setup(41, seq_lens, n_q, dtype)
    total = int(sum(seq_lens))
    pool_a, pool_b = pool.clone(), pool.clone()
    for r, s in enumerate(seq_lens):   # reference path: append, then decode
        ctx.encode_append(pool_a, tabs[r], s - n_q, k_new[r], v_new[r])
    out_a = ctx.decode_attention(pool_a, q, tabs, seq, total, SCALE)
    out_b = ctx.decode_append_attention(pool_b, k_new, v_new, q, tabs, seq, total, SCALE)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    assert torch.equal(pool_a, pool_b), "pool bytes differ"
    assert torch.equal(out_a, out_b), "outputs differ"


def test_fused_append_against_oracle():
    n_q, seq_lens = 1, [3000]
    ctx, signs, pool, tab, tabs, k_new, v_new, q, qb, seq, hist = _setup(43, seq_lens, n_q, torch.float32)
    out = ctx.decode_append_attention(pool, k_new, v_new, q, tabs, seq, 3000, SCALE, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    c, _ = O.codebook()
    # the oracle reads the GPU's pool bytes (history and the fused append alike)
    exp = O.decode_attention(pool.cpu().numpy(), tab, np.array(seq_lens),
                             I.bf16_bits_to_f32(qb).astype(np.float64), SCALE, signs, c)
    got = out.cpu().numpy().astype(np.float64)
    assert np.abs(got - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())
    # and the appended position is the oracle's own encoding of the new vectors
    opool = O.new_pool(pool.numel() // O.PAGE_BYTES)
    yk, yv = O.encode_append(opool, tab[0], 2999, hist[0][0][2999:], hist[0][1][2999:], signs, c)
    gk, gv, gkn, gvn = O._regions(pool.cpu().numpy())
    ok_, ov_, okn, ovn = O._regions(opool)
    pg, sl = tab[0][2999 // 256], 2999 % 256
    _, b = O.codebook()
    H.check_words_against_oracle(gk[pg, :, sl][None], ok_[pg, :, sl][None], yk, b, "K words")
    H.check_words_against_oracle(gv[pg, :, sl][None], ov_[pg, :, sl][None], yv, b, "V words")


def test_fused_append_rejects_bad_arguments():
    ctx = tq4.Context(I.signs(41))
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    rc = tq4.tq4_decode_append_attention(ctx.handle, dummy, 1, None, dummy, tq4.DTYPE_F32, dummy, dummy, 1,
                                         dummy, 1, 1, 1, SCALE, dummy, tq4.DTYPE_BF16, dummy, 256)
    assert rc == tq4.TQ4_ERR_ARG
    rc = tq4.tq4_decode_append_attention(ctx.handle, dummy, 1, dummy, dummy, 7, dummy, dummy, 1,
                                         dummy, 1, 1, 1, SCALE, dummy, tq4.DTYPE_BF16, dummy, 256)
    assert rc == tq4.TQ4_ERR_ARG
