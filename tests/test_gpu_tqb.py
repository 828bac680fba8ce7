"""GPU parity of the 2- and 3-bit variants against their fp64 oracle
(oracle/tqb_oracle.py), through the C ABI: the library's codebooks equal the
oracle's; the encode is bit-exact apart from coordinates within 1e-6 of a decision
boundary (the GPU rotates in fp32); decode attention meets the bf16 tolerance on the
GPU-encoded pool and 1e-4 (fp32 output) on the oracle's own pool bytes, for one to
four query tokens, ragged lengths, shared pages, outliers and a 32,768-position
history."""
import numpy as np
import pytest

from compressed_paged_kv_tq4_b200 import inputs as I
from oracle import tqb_oracle as OB
import _helpers as H

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from compressed_paged_kv_tq4_b200 import tq4  # noqa: E402

SCALE = 1.0 / 16.0


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("bits", [2, 3])
def test_tqb_codebook_matches_oracle(bits):
    ctx = tq4.Context(I.signs(0))
    c, b = ctx.tqb_codebook(bits)
    oc, ob = OB.codebook(bits)
    assert np.max(np.abs(np.array(c) - oc)) < 1e-15
    assert np.max(np.abs(np.array(b) - ob)) < 1e-15


def _pool_regions(pool_bytes, bits):
    return OB._regions(np.ascontiguousarray(pool_bytes), bits)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tqb_encode_bit_exact(bits, dtype):
    signs = I.signs(0)
    ctx = tq4.Context(signs)
    c, b = OB.codebook(bits)
    table = I.page_table_scattered(41, 5, 7)
    k, v = I.kv_vectors(41, 0, 1200, outlier_frac=0.05)
    k[17] = 0.0                                        # a zero vector
    if dtype == "bf16":
        kb, vb = I.to_bf16_bits(k), I.to_bf16_bits(v)
        k, v = I.bf16_bits_to_f32(kb), I.bf16_bits_to_f32(vb)
        kt, vt = _bf16_tensor(kb), _bf16_tensor(vb)
    else:
        kt, vt = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    pool = tq4.Context.new_tqb_pool(bits, 7)
    tt = torch.from_numpy(table).cuda()
    for a, e in ((0, 333), (333, 1000), (1000, 1200)):   # appends that start mid-page
        ctx.tqb_encode_append(bits, pool, tt, a, kt[a:e], vt[a:e])
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    opool = OB.new_pool(7, bits)
    yk, yv = OB.encode_append(opool, table, 0, k, v, signs, c, bits)
    g = _pool_regions(pool.cpu().numpy(), bits)
    o = _pool_regions(opool, bits)
    pos = np.arange(1200)
    pg, sl = table[pos // 256], pos % 256
    exempt = 0
    for gw, ow, y, what in ((g[0], o[0], yk, "K"), (g[1], o[1], yv, "V")):
        gi = OB.unpack_indices(gw[pg, :, sl], bits).astype(np.int64)
        oi = OB.unpack_indices(ow[pg, :, sl], bits).astype(np.int64)
        diff = gi != oi
        if diff.any():
            dist = np.min(np.abs(np.asarray(y)[diff][:, None] - b[None, :]), axis=1)
            ok = (dist < H.BOUNDARY_EXEMPT) & (np.abs(gi[diff] - oi[diff]) == 1)
            assert ok.all(), f"{what}: {int((~ok).sum())} indices differ away from a boundary"
            exempt += int(diff.sum())
        # every word bit outside the differing indices is identical: repack the oracle's
        # indices with the GPU's exempt ones and compare the words
        fixed = np.where(diff, gi, oi).astype(np.uint8)
        assert np.array_equal(OB.pack_indices(fixed, bits), gw[pg, :, sl])
    assert exempt <= 20
    H.check_norms_against_oracle(g[2][pg, :, sl], o[2][pg, :, sl], k, "K norms")
    H.check_norms_against_oracle(g[3][pg, :, sl], o[3][pg, :, sl], v, "V norms")


class TqbCase:
    def __init__(self, bits, config, seq_lens, n_q, shared_pages=0, outliers=0.05, hist=None):
        """Pools (GPU-encoded and oracle-encoded) whose tables cover seq_lens; the
        first hist[r] positions of request r are encoded (all of them by default)."""
        self.bits = bits
        self.signs = I.signs(config)
        self.ctx = tq4.Context(self.signs)
        self.c, _ = OB.codebook(bits)
        npg = [(s + 255) // 256 for s in seq_lens]
        total = npg[0] + sum(n - shared_pages for n in npg[1:]) + 2
        ids = I.page_table_scattered(config, total, total)
        tab = np.full((len(seq_lens), max(npg)), -1, np.int32)
        tab[0, :npg[0]] = ids[:npg[0]]
        off = npg[0]
        for r in range(1, len(seq_lens)):
            tab[r, :shared_pages] = tab[0, :shared_pages]
            f = npg[r] - shared_pages
            tab[r, shared_pages:npg[r]] = ids[off:off + f]
            off += f
        self.tab, self.n_q = tab, n_q
        self.seq = np.array(seq_lens, np.int32)
        self.pool = tq4.Context.new_tqb_pool(bits, total)
        self.opool = OB.new_pool(total, bits)
        for r, s in enumerate(seq_lens if hist is None else hist):
            first = shared_pages * 256 if r > 0 else 0
            k, v = I.kv_vectors(config, 0, s - first, first_pos=first, request=r, outlier_frac=outliers)
            self.ctx.tqb_encode_append(bits, self.pool, torch.from_numpy(tab[r]).cuda(), first,
                                       torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            OB.encode_append(self.opool, tab[r], first, k, v, self.signs, self.c, bits)
        torch.cuda.synchronize()
        assert self.ctx.status() == tq4.TQ4_OK

    def decode(self, qb, pool, out_dtype):
        out = self.ctx.tqb_decode_attention(self.bits, pool, _bf16_tensor(qb), torch.from_numpy(self.tab).cuda(),
                                            torch.from_numpy(self.seq).cuda(), int(self.seq.sum()), SCALE,
                                            out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert self.ctx.status() == tq4.TQ4_OK
        return out.float().cpu().numpy().astype(np.float64)

    def oracle(self, qb):
        return OB.decode_attention(self.opool, self.tab, self.seq, I.bf16_bits_to_f32(qb), SCALE, self.signs,
                                   self.c, self.bits)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("seq_lens,n_q,shared", [
    ([1], 1, 0), ([255], 1, 0), ([257], 1, 0), ([1000, 63, 2047], 1, 0), ([300], 2, 0),
    ([513, 40], 3, 0), ([2048, 700], 4, 2), ([4], 4, 0), ([5000], 4, 0),
])
def test_tqb_decode_parity(bits, seq_lens, n_q, shared):
    case = TqbCase(bits, 43, seq_lens, n_q, shared_pages=shared)
    qb = I.queries(43, 1, (len(seq_lens), n_q, 24, 256))
    exp = case.oracle(qb)
    H.assert_bf16_close(case.decode(qb, case.pool, torch.bfloat16), exp, f"{bits}-bit decode {seq_lens} n_q={n_q}")
    got32 = case.decode(qb, torch.from_numpy(case.opool).cuda(), torch.float32)
    assert np.abs(got32 - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())


@pytest.mark.parametrize("bits", [2, 3])
def test_tqb_decode_32k_history(bits):
    """The decode_32k shape (one request, 32,768 positions, one query token)."""
    case = TqbCase(bits, 44, [32768], 1, outliers=0.0)
    qb = I.queries(44, 0, (1, 1, 24, 256))
    exp = case.oracle(qb)
    got32 = case.decode(qb, torch.from_numpy(case.opool).cuda(), torch.float32)
    assert np.abs(got32 - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())
    H.assert_bf16_close(case.decode(qb, case.pool, torch.bfloat16), exp, f"{bits}-bit decode 32k")


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("seq_lens,n_q,new_dtype", [
    ([3000], 1, "f32"),                 # one token, fused into the one-token decode kernel
    ([257, 1000, 64], 1, "bf16"),       # position 256 opens a page; three requests
    ([2000, 700], 4, "f32"),            # four tokens: the tail-encode kernel, then the decode
])
def test_tqb_fused_append(bits, seq_lens, n_q, new_dtype):
    """tq4_tqb_decode_append_attention writes the same pool bytes as a separate
    tq4_tqb_encode_append and then returns the same output as tq4_tqb_decode_attention
    (the same kernels on the same bytes: bit-identical); against the oracle, which
    encodes the new tokens itself, within the bf16 tolerance."""
    hist = [s - n_q for s in seq_lens]
    case = TqbCase(bits, 45, seq_lens, n_q, hist=hist)
    dt = torch.float32 if new_dtype == "f32" else torch.bfloat16
    k_new, v_new = [], []
    for r, s in enumerate(hist):
        k, v = I.kv_vectors(45, 1, n_q, first_pos=s, request=r)
        k_new.append(k)
        v_new.append(v)
    kn = np.stack(k_new)
    vn = np.stack(v_new)
    kt = torch.from_numpy(kn).cuda().to(dt)
    vt = torch.from_numpy(vn).cuda().to(dt)
    qb = I.queries(45, 2, (len(seq_lens), n_q, 24, 256))
    tab = torch.from_numpy(case.tab).cuda()
    seq = torch.from_numpy(case.seq).cuda()
    pool_b = case.pool.clone()
    fused = case.ctx.tqb_decode_append_attention(bits, case.pool, kt, vt, _bf16_tensor(qb), tab, seq,
                                                 int(case.seq.sum()), SCALE, out_dtype=torch.float32)
    for r, s in enumerate(hist):
        case.ctx.tqb_encode_append(bits, pool_b, tab[r], s, kt[r], vt[r])
    plain = case.ctx.tqb_decode_attention(bits, pool_b, _bf16_tensor(qb), tab, seq, int(case.seq.sum()), SCALE,
                                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_OK
    assert torch.equal(case.pool, pool_b)
    assert torch.equal(fused, plain)
    for r, s in enumerate(hist):   # the oracle's pool gets the new tokens as the GPU saw them
        k = kt[r].float().cpu().numpy().astype(np.float64)
        v = vt[r].float().cpu().numpy().astype(np.float64)
        OB.encode_append(case.opool, case.tab[r], s, k, v, case.signs, case.c, bits)
    H.assert_bf16_close(fused.cpu().numpy().astype(np.float64), case.oracle(qb),
                        f"{bits}-bit fused append {seq_lens} n_q={n_q}")


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("seq_lens,n_q,shared,leader", [
    ([3000, 2500, 4000], 1, 8, [0, 0, 0]),            # one group of three, one token
    ([3000, 700, 2900, 5000], 2, 2, [0, 0, 0, 3]),    # a group of three; request 3 alone
    ([2600, 2600, 2700], 4, 8, [0, 0, 0]),            # three four-token members: cut to 2 + 1
])
def test_tqb_shared_prefix_parity(bits, seq_lens, n_q, shared, leader):
    """Shared-prefix groups over a b-bit pool (shared pages read and widened once for
    every member). The attention arithmetic is checked on the oracle's own pool bytes
    (bf16 tolerance, and 1e-4 in fp32): the GPU-encoded pool may differ from the
    oracle's where the spec exempts it (a coordinate within 1e-6 of a decision
    boundary, a norm at an fp16 rounding midpoint), and in these seeded requests one
    such norm, of a x8 outlier key that dominates a token's attention, moves that
    token's output by more than a bf16 ulp. On the GPU-encoded pool the grouped
    decode must equal the ungrouped one within fp32 summation order."""
    case = TqbCase(bits, 47, seq_lens, n_q, shared_pages=shared)
    pages = [shared if leader[r] == 0 else 0 for r in range(len(seq_lens))]
    qb = I.queries(47, 0, (len(seq_lens), n_q, 24, 256))
    exp = case.oracle(qb)
    tab = torch.from_numpy(case.tab).cuda()
    seq = torch.from_numpy(case.seq).cuda()
    opool = torch.from_numpy(case.opool).cuda()

    def shared_decode(pool, out_dtype):
        return case.ctx.tqb_decode_attention_shared(bits, pool, _bf16_tensor(qb), tab, seq, int(case.seq.sum()),
                                                    SCALE, leader, pages, out_dtype=out_dtype)
    got16 = shared_decode(opool, torch.bfloat16)
    got32 = shared_decode(opool, torch.float32)
    grouped = shared_decode(case.pool, torch.float32)
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_OK
    H.assert_bf16_close(got16.float().cpu().numpy(), exp, f"{bits}-bit shared prefix {seq_lens} n_q={n_q}")
    g32 = got32.cpu().numpy().astype(np.float64)
    assert np.abs(g32 - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())
    plain = case.decode(qb, case.pool, torch.float32)
    gg = grouped.cpu().numpy().astype(np.float64)
    assert np.abs(gg - plain).max() <= 1e-5 * max(1.0, np.abs(plain).max())


@pytest.mark.parametrize("bits", [2, 3])
def test_tqb_reconstruct_matches_oracle(bits):
    """Explicit K/V from the oracle's own b-bit pool bytes against the oracle's
    reconstruction (per vector, relative), over scattered pages and a ragged range."""
    c, _ = OB.codebook(bits)
    signs = I.signs(1)
    ctx = tq4.Context(signs)
    table = np.array([3, 0, 2], np.int32)
    k, v = I.kv_vectors(1, 1, 700, outlier_frac=0.05)
    opool = OB.new_pool(4, bits)
    OB.encode_append(opool, table, 0, k, v, signs, c, bits)
    kr, vr = ctx.tqb_reconstruct(bits, torch.from_numpy(opool).cuda(), torch.from_numpy(table).cuda(), 5, 690)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    ko, vo = OB.reconstruct(opool, table, 5, 690, signs, c, bits)
    for got, exp in ((kr.cpu().numpy(), ko), (vr.cpu().numpy(), vo)):
        rel = np.linalg.norm(got - exp, axis=-1) / np.maximum(np.linalg.norm(exp, axis=-1), 1e-30)
        assert rel.max() < 1e-6, rel.max()


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("prefix_len,n_tok,outliers", [
    (0, 40, 0.0), (300, 100, 0.05), (1000, 257, 0.0), (4096, 64, 0.05),
])
def test_tqb_prefill_parity(bits, prefix_len, n_tok, outliers):
    """The prefill over a b-bit prefix (rebuilt as dense rows, then the tcgen05
    attention) against the b-bit oracle: every row, bf16 on the GPU-encoded pool and
    1e-4 in fp32 on the oracle's own pool bytes."""
    c, _ = OB.codebook(bits)
    signs = I.signs(5)
    ctx = tq4.Context(signs)
    npg = max(1, (prefix_len + 255) // 256)
    table = I.page_table_scattered(5, npg, npg + 2)
    tt = torch.from_numpy(table).cuda()
    pool = tq4.Context.new_tqb_pool(bits, npg + 2)
    opool = OB.new_pool(npg + 2, bits)
    if prefix_len:
        k, v = I.kv_vectors(5, 0, prefix_len, outlier_frac=outliers)
        ctx.tqb_encode_append(bits, pool, tt, 0, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        OB.encode_append(opool, table, 0, k, v, signs, c, bits)
    qb = I.queries(5, 0, (n_tok, 24, 256))
    kb, vb = I.chunk_kv(5, 0, n_tok)
    args = (_bf16_tensor(qb), _bf16_tensor(kb), _bf16_tensor(vb), SCALE)
    out = ctx.tqb_prefill_attention(bits, pool, tt, prefix_len, *args)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    exp = OB.prefill_attention(opool, table, prefix_len, I.bf16_bits_to_f32(qb), I.bf16_bits_to_f32(kb),
                               I.bf16_bits_to_f32(vb), SCALE, signs, c, bits)
    H.assert_bf16_close(out.float().cpu().numpy(), exp, f"{bits}-bit prefill {prefix_len}+{n_tok}")
    out32 = ctx.tqb_prefill_attention(bits, torch.from_numpy(opool).cuda(), tt, prefix_len, *args,
                                      out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    err = np.abs(out32.cpu().numpy().astype(np.float64) - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), (bits, prefix_len, n_tok, err)


@pytest.mark.parametrize("bits", [2, 3])
def test_tqb_prefill_2k_on_32k_sampled(bits):
    """The prefill workload's shape (2,048 chunk tokens on a 32,768-position prefix) over a
    b-bit pool, checked on sampled chunk tokens (first and last included)."""
    c, _ = OB.codebook(bits)
    signs = I.signs(6)
    ctx = tq4.Context(signs)
    prefix_len, n_tok = 32768, 2048
    npg = prefix_len // 256
    table = I.page_table_scattered(6, npg, npg + 8)
    tt = torch.from_numpy(table).cuda()
    k, v = I.kv_vectors(6, 0, prefix_len)
    pool = tq4.Context.new_tqb_pool(bits, npg + 8)
    opool = OB.new_pool(npg + 8, bits)
    ctx.tqb_encode_append(bits, pool, tt, 0, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    OB.encode_append(opool, table, 0, k, v, signs, c, bits)
    qb = I.queries(6, 0, (n_tok, 24, 256))
    kb, vb = I.chunk_kv(6, 0, n_tok)
    rows = np.array([0, 1, 255, 256, 1023, 1500, 2046, 2047])
    out = ctx.tqb_prefill_attention(bits, torch.from_numpy(opool).cuda(), tt, prefix_len, _bf16_tensor(qb),
                                    _bf16_tensor(kb), _bf16_tensor(vb), SCALE, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    exp = OB.prefill_attention(opool, table, prefix_len, I.bf16_bits_to_f32(qb), I.bf16_bits_to_f32(kb),
                               I.bf16_bits_to_f32(vb), SCALE, signs, c, bits, rows=rows)
    got = out.cpu().numpy().astype(np.float64)[rows]
    assert np.abs(got - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())


@pytest.mark.parametrize("bits", [2, 3])
def test_tqb_bad_page_id(bits):
    """A page id outside the pool is reported (TQ4_ERR_PAGE_RANGE) by the encode, the
    one-token decode and the fused step, and nothing is written outside the pool's
    valid pages: page 1, which the table never names, stays zero."""
    ctx = tq4.Context(I.signs(0))
    pool = tq4.Context.new_tqb_pool(bits, 2)
    table = torch.tensor([0, 7], dtype=torch.int32, device="cuda")   # 7 is outside a 2-page pool
    k = torch.randn(300, 4, 256, device="cuda")
    ctx.tqb_encode_append(bits, pool, table, 0, k, k)
    assert ctx.status() == tq4.TQ4_ERR_PAGE_RANGE
    assert ctx.status() == tq4.TQ4_OK   # cleared by the read
    page_bytes = tq4.TQB_PAGE_BYTES[bits]
    assert int(pool[page_bytes:].sum()) == 0
    q = torch.zeros(1, 1, 24, 256, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([300], dtype=torch.int32, device="cuda")
    ctx.tqb_decode_attention(bits, pool, q, table[None], seq, 300, SCALE)
    assert ctx.status() == tq4.TQ4_ERR_PAGE_RANGE
    kn = torch.randn(1, 1, 4, 256, device="cuda")
    ctx.tqb_decode_append_attention(bits, pool, kn, kn, q, table[None], seq, 300, SCALE)
    assert ctx.status() == tq4.TQ4_ERR_PAGE_RANGE
    assert int(pool[page_bytes:].sum()) == 0


def test_tqb_argument_checks():
    ctx = tq4.Context(I.signs(0))
    assert tq4.tq4_tqb_encode_append(ctx.handle, 4, None, 1, None, 1, 0, 1, None, None, 1) == tq4.TQ4_ERR_UNSUPPORTED
    assert tq4.tq4_tqb_decode_attention(ctx.handle, 5, None, 1, None, None, 1, None, 1, 1, 1, SCALE, None, 1,
                                        None, 0) == tq4.TQ4_ERR_UNSUPPORTED
