"""GPU parity at sizes the oracle finishes in seconds: the CUDA path (through
the C ABI) against the fp64 oracle on the same seeded inputs."""
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


def _pool_view(pool_bytes):
    pages = pool_bytes.reshape(-1, O.PAGE_BYTES)
    kw = pages[:, 0:131072].view("<u4").reshape(-1, 4, 256, 32)
    vw = pages[:, 131072:262144].view("<u4").reshape(-1, 4, 256, 32)
    kn = pages[:, 262144:264192].view("<f2").reshape(-1, 4, 256)
    vn = pages[:, 264192:266240].view("<f2").reshape(-1, 4, 256)
    return kw, vw, kn, vn


@pytest.fixture(scope="module")
def codebook():
    return O.codebook()


class Case:
    """One small problem built identically on the GPU and in the oracle."""

    def __init__(self, config, seq_lens, n_q, shared_pages=0, outliers=0.0, chunks=(1000,)):
        self.signs = I.signs(config)
        self.ctx = tq4.Context(self.signs)
        self.c, self.b = O.codebook()
        npg = [(s + 255) // 256 for s in seq_lens]
        total_pages = npg[0] + sum(n - shared_pages for n in npg[1:]) + 3
        ids = I.page_table_scattered(config, total_pages, total_pages)
        tab = np.full((len(seq_lens), max(npg)), -1, np.int32)
        tab[0, :npg[0]] = ids[:npg[0]]
        off = npg[0]
        for r in range(1, len(seq_lens)):
            tab[r, :shared_pages] = tab[0, :shared_pages]
            f = npg[r] - shared_pages
            tab[r, shared_pages:npg[r]] = ids[off:off + f]
            off += f
        self.tab = tab
        self.num_pages = total_pages
        self.seq_lens = np.array(seq_lens, np.int32)
        self.n_q = n_q
        self.pool = tq4.Context.new_pool(total_pages)
        self.opool = O.new_pool(total_pages)
        self.kv = []
        for r, s in enumerate(seq_lens):
            first = shared_pages * 256 if r > 0 else 0
            k, v = I.kv_vectors(config, 0, s - first, first_pos=first, request=r, outlier_frac=outliers)
            self.kv.append((first, k, v))
            tt = torch.from_numpy(tab[r]).cuda()
            pos, i = 0, 0
            while pos < k.shape[0]:  # ragged appends, sizes cycling through `chunks`
                n = min(chunks[i % len(chunks)], k.shape[0] - pos)
                self.ctx.encode_append(self.pool, tt, first + pos, torch.from_numpy(k[pos:pos + n]).cuda(),
                                       torch.from_numpy(v[pos:pos + n]).cuda())
                pos, i = pos + n, i + 1
            O.encode_append(self.opool, tab[r], first, k, v, self.signs, self.c)
        torch.cuda.synchronize()
        assert self.ctx.status() == tq4.TQ4_OK

    def decode(self, q_bits, out_dtype=torch.bfloat16):
        q = _bf16_tensor(q_bits)
        out = self.ctx.decode_attention(self.pool, q, torch.from_numpy(self.tab).cuda(),
                                        torch.from_numpy(self.seq_lens).cuda(), int(self.seq_lens.sum()),
                                        SCALE, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert self.ctx.status() == tq4.TQ4_OK
        return out.float().cpu().numpy()

    def decode_oracle_pool(self, q_bits, out_dtype=torch.float32):
        """GPU decode over the oracle's pool bytes: identical packed inputs on both sides."""
        q = _bf16_tensor(q_bits)
        opool = torch.from_numpy(self.opool).cuda()
        out = self.ctx.decode_attention(opool, q, torch.from_numpy(self.tab).cuda(),
                                        torch.from_numpy(self.seq_lens).cuda(), int(self.seq_lens.sum()),
                                        SCALE, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert self.ctx.status() == tq4.TQ4_OK
        return out.float().cpu().numpy()

    def oracle_decode(self, q_bits):
        qf = I.bf16_bits_to_f32(q_bits).astype(np.float64)
        return O.decode_attention(self.opool, self.tab, self.seq_lens, qf, SCALE, self.signs, self.c)


def test_library_codebook_matches_oracle(codebook):
    ctx = tq4.Context(I.signs(0))
    c, b = ctx.codebook()
    assert np.max(np.abs(np.array(c) - codebook[0])) < 1e-15
    assert np.max(np.abs(np.array(b) - codebook[1])) < 1e-15


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_encode_append_bit_exact(codebook, dtype):
    c, b = codebook
    signs = I.signs(0)
    ctx = tq4.Context(signs)
    w = I.WORKLOADS["single_layer_2k"]
    table = I.request_tables(w)[0]
    k, v = I.kv_vectors(0, 0, 2048)
    if dtype == "bf16":
        kb, vb = I.to_bf16_bits(k), I.to_bf16_bits(v)
        k, v = I.bf16_bits_to_f32(kb), I.bf16_bits_to_f32(vb)
        kt, vt = _bf16_tensor(kb), _bf16_tensor(vb)
    else:
        kt, vt = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    pool = tq4.Context.new_pool(8)
    tt = torch.from_numpy(table).cuda()
    for a, e in ((0, 700), (700, 1537), (1537, 2048)):  # appends that start mid-page
        ctx.encode_append(pool, tt, a, kt[a:e], vt[a:e])
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    opool = O.new_pool(8)
    yk, yv = O.encode_append(opool, table, 0, k, v, signs, c)
    gkw, gvw, gkn, gvn = _pool_view(pool.cpu().numpy())
    okw, ovw, okn, ovn = _pool_view(opool)
    pos = np.arange(2048)
    pg, sl = table[pos // 256], pos % 256
    nk = H.check_words_against_oracle(gkw[pg, :, sl], okw[pg, :, sl], yk, b, "K words")
    nv = H.check_words_against_oracle(gvw[pg, :, sl], ovw[pg, :, sl], yv, b, "V words")
    H.check_norms_against_oracle(gkn[pg, :, sl], okn[pg, :, sl], k, "K norms")
    H.check_norms_against_oracle(gvn[pg, :, sl], ovn[pg, :, sl], v, "V norms")
    assert nk + nv <= 20  # a handful of exempt boundary nibbles out of 4.2M


def test_reconstruct_matches_oracle(codebook):
    """GPU reconstruction of the oracle's own pool bytes against the oracle's reconstruction."""
    c, _ = codebook
    signs = I.signs(0)
    ctx = tq4.Context(signs)
    table = np.array([3, 0, 2], np.int32)
    k, v = I.kv_vectors(0, 1, 700, outlier_frac=0.05)
    opool = O.new_pool(4)
    O.encode_append(opool, table, 0, k, v, signs, c)
    kr, vr = ctx.reconstruct(torch.from_numpy(opool).cuda(), torch.from_numpy(table).cuda(), 5, 690)
    ko, vo = O.reconstruct(opool, table, 5, 690, signs, c)
    for got, exp in ((kr.cpu().numpy(), ko), (vr.cpu().numpy(), vo)):
        rel = np.linalg.norm(got - exp, axis=-1) / np.maximum(np.linalg.norm(exp, axis=-1), 1e-30)
        assert rel.max() < H.RECON_REL_TOL
        assert rel.max() < 1e-6  # fp32 arithmetic: far inside the stated bound


def test_decode_single_layer_2k_parity():
    case = Case(0, [2048], 1)
    q = I.queries(0, 0, (1, 1, 24, 256))
    got = case.decode(q)
    exp = case.oracle_decode(q)
    H.assert_bf16_close(got, exp, "bf16 out")
    # attention arithmetic alone: same packed bytes on both sides, fp32 output
    got32 = case.decode_oracle_pool(q)
    err = np.abs(got32 - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), err


@pytest.mark.parametrize("seq_lens,n_q,shared", [
    ([1], 1, 0), ([17], 1, 0), ([255], 1, 0), ([256], 1, 0), ([257], 1, 0),
    ([1000, 63, 2047], 1, 0), ([300], 2, 0), ([513, 40], 3, 0), ([2048, 700], 4, 2),
    ([4], 4, 0), ([5000], 4, 0),
    # one query token, longer splits: full rounds of 32-position tiles, then 16-position
    # tail tiles (remainder <= 128) or a partial round of 32-position tiles (remainder > 128)
    ([20000], 1, 0), ([9000, 3100], 1, 0),
])
def test_decode_variants_parity(seq_lens, n_q, shared):
    case = Case(7, seq_lens, n_q, shared_pages=shared, outliers=0.05, chunks=(333,))
    q = I.queries(7, 1, (len(seq_lens), n_q, 24, 256))
    got = case.decode(q)
    exp = case.oracle_decode(q)
    H.assert_bf16_close(got, exp, f"decode {seq_lens} n_q={n_q}")
    # the attention arithmetic in fp32 on the oracle's own pool bytes (5% x8 outliers)
    got32 = case.decode_oracle_pool(q)
    err = np.abs(got32 - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), err


@pytest.mark.parametrize("n_q", [1, 4])
def test_decode_split_count_invariance(n_q):
    """The host bound total_seq_len sets the split length: a looser bound gives fewer,
    longer splits. Both plans must give the same attention (fp32 outputs, to the fp32
    tolerance), and both must match the oracle."""
    case = Case(11, [5000], n_q, outliers=0.05, chunks=(777,))
    q = I.queries(11, 0, (1, n_q, 24, 256))
    qt = _bf16_tensor(q)
    pool = torch.from_numpy(case.opool).cuda()
    width = 160                                  # table wider than the request: room for a loose bound
    tab = np.full((1, width), -1, np.int32)
    tab[0, :case.tab.shape[1]] = case.tab[0]
    tt, seq = torch.from_numpy(tab).cuda(), torch.from_numpy(case.seq_lens).cuda()
    outs = []
    for total in (5000, width * 256):            # 20 splits of 256 positions, then 5 of 1,152
        outs.append(case.ctx.decode_attention(pool, qt, tt, seq, total, SCALE, out_dtype=torch.float32)
                    .cpu().numpy())
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_OK
    exp = case.oracle_decode(q)
    tol = H.F32_ABS_TOL * max(1.0, np.abs(exp).max())
    assert np.abs(outs[0] - outs[1]).max() <= tol
    for got in outs:
        assert np.abs(got - exp).max() <= tol


def test_decode_first_of_four_tokens_equals_one_token_decode():
    """Causal verify: query token 0 of an n_q = 4 call at length T sees [0, T-4], the
    same history as a one-token call at length T-3 with the same query (fp32 outputs,
    identical pool bytes; the two calls run different kernels)."""
    case = Case(12, [3001], 4, outliers=0.05)
    q4 = I.queries(12, 0, (1, 4, 24, 256))
    pool = torch.from_numpy(case.opool).cuda()
    tt = torch.from_numpy(case.tab).cuda()
    out4 = case.ctx.decode_attention(pool, _bf16_tensor(q4), tt, torch.tensor([3001], dtype=torch.int32,
                                     device="cuda"), 3001, SCALE, out_dtype=torch.float32).cpu().numpy()
    out1 = case.ctx.decode_attention(pool, _bf16_tensor(np.ascontiguousarray(q4[:, :1])), tt,
                                     torch.tensor([2998], dtype=torch.int32, device="cuda"), 2998, SCALE,
                                     out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_OK
    tol = H.F32_ABS_TOL * max(1.0, np.abs(out1).max())
    assert np.abs(out4[:, 0] - out1[:, 0]).max() <= tol


def test_decode_page_table_permutation_invariance():
    """The same logical history through two different page tables gives identical GPU output."""
    ctx = tq4.Context(I.signs(8))
    k, v = I.kv_vectors(8, 0, 1500)
    q = _bf16_tensor(I.queries(8, 0, (1, 1, 24, 256)))
    seq = torch.tensor([1500], dtype=torch.int32, device="cuda")
    outs = []
    for salt in (0, 1):
        table = I.page_table_scattered(8, 6, 9, salt=salt)
        pool = tq4.Context.new_pool(9)
        tt = torch.from_numpy(table).cuda()
        ctx.encode_append(pool, tt, 0, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        outs.append(ctx.decode_attention(pool, q, tt[None], seq, 1500, SCALE).cpu())
    assert ctx.status() == tq4.TQ4_OK
    assert not np.array_equal(I.page_table_scattered(8, 6, 9, salt=0), I.page_table_scattered(8, 6, 9, salt=1))
    assert torch.equal(outs[0], outs[1])


# (prefix_len, n_tok, outlier_frac): one or several 128-row blocks per KV head with a
# ragged last block; prefixes that end inside a 64-position tile and cross pages;
# 5% x8 outlier norms, whose large scores raise the softmax reference mid-walk. Both
# prefill paths: the prefix expanded from packed words inside the attention kernel,
# and rebuilt as dense rows first (direct inverse reconstruction)
@pytest.mark.parametrize("reconstruct", [False, True])
@pytest.mark.parametrize("prefix_len,n_tok,outliers", [(300, 70, 0.0), (0, 5, 0.0), (512, 64, 0.0), (1, 1, 0.0),
                                                       (777, 130, 0.0), (1000, 200, 0.0), (600, 43, 0.05),
                                                       (2048, 22, 0.05), (1500, 90, 0.05), (64, 300, 0.0)])
def test_prefill_parity(codebook, prefix_len, n_tok, outliers, reconstruct):
    c, _ = codebook
    signs = I.signs(4)
    ctx = tq4.Context(signs)
    npg = max(1, (prefix_len + 255) // 256)
    table = I.page_table_scattered(4, npg, npg + 2)
    k, v = I.kv_vectors(4, 0, prefix_len, outlier_frac=outliers)
    pool = tq4.Context.new_pool(npg + 2)
    tt = torch.from_numpy(table).cuda()
    if prefix_len:
        ctx.encode_append(pool, tt, 0, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    opool = O.new_pool(npg + 2)
    if prefix_len:
        O.encode_append(opool, table, 0, k, v, signs, c)
    qb = I.queries(4, 0, (n_tok, 24, 256))
    kb, vb = I.chunk_kv(4, 0, n_tok)
    out = ctx.prefill_attention(pool, tt, prefix_len, _bf16_tensor(qb), _bf16_tensor(kb), _bf16_tensor(vb), SCALE,
                                reconstruct=reconstruct)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    exp = O.prefill_attention(opool, table, prefix_len, I.bf16_bits_to_f32(qb), I.bf16_bits_to_f32(kb),
                              I.bf16_bits_to_f32(vb), SCALE, signs, c)
    H.assert_bf16_close(out.float().cpu().numpy(), exp, f"prefill {prefix_len}+{n_tok} outliers {outliers}")
    # fp32 output on the oracle's own pool bytes: the attention arithmetic alone, every row
    out32 = ctx.prefill_attention(torch.from_numpy(opool).cuda(), tt, prefix_len, _bf16_tensor(qb), _bf16_tensor(kb),
                                  _bf16_tensor(vb), SCALE, out_dtype=torch.float32, reconstruct=reconstruct)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    err = np.abs(out32.cpu().numpy().astype(np.float64) - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), (prefix_len, n_tok, outliers, err)
    if reconstruct:   # the two paths compute the same values (fp32, up to rounding order)
        other = ctx.prefill_attention(torch.from_numpy(opool).cuda(), tt, prefix_len, _bf16_tensor(qb),
                                      _bf16_tensor(kb), _bf16_tensor(vb), SCALE, out_dtype=torch.float32)
        torch.cuda.synchronize()
        diff = (out32 - other).abs().max().item()
        assert diff <= 2e-5 * max(1.0, other.abs().max().item()), diff


# ------------------------------------------------------------------ failure paths (no GPU fault)
def test_bad_page_id_is_recorded_not_faulted():
    ctx = tq4.Context(I.signs(0))
    pool = tq4.Context.new_pool(2)
    table = torch.tensor([0, 7], dtype=torch.int32, device="cuda")   # 7 is outside a 2-page pool
    k = torch.randn(300, 4, 256, device="cuda")
    ctx.encode_append(pool, table, 0, k, k)
    assert ctx.status() == tq4.TQ4_ERR_PAGE_RANGE
    assert ctx.status() == tq4.TQ4_OK  # cleared by the read
    q = torch.zeros(1, 1, 24, 256, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([300], dtype=torch.int32, device="cuda")
    ctx.decode_attention(pool, q, table[None], seq, 300, SCALE)
    assert ctx.status() == tq4.TQ4_ERR_PAGE_RANGE


def test_host_side_argument_errors():
    ctx = tq4.Context(I.signs(0))
    pool = tq4.Context.new_pool(1)
    table = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    seq = torch.tensor([10], dtype=torch.int32, device="cuda")
    q5 = torch.zeros(1, 5, 24, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq4.TQ4Error) as e:
        ctx.decode_attention(pool, q5, table, seq, 10, SCALE)
    assert e.value.code == tq4.TQ4_ERR_UNSUPPORTED
    q = torch.zeros(1, 1, 24, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq4.TQ4Error) as e:
        ctx.decode_attention(pool, q, table, seq, 10, SCALE,
                             workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert e.value.code == tq4.TQ4_ERR_WORKSPACE
    with pytest.raises(tq4.TQ4Error) as e:   # more positions than the table can hold
        ctx.decode_attention(pool, q, table, seq, 10_000, SCALE)
    assert e.value.code == tq4.TQ4_ERR_ARG
    rc = tq4.tq4_encode_append(ctx.handle, pool, 1, table, 1, 250, 10, q, q, tq4.DTYPE_BF16)
    assert rc == tq4.TQ4_ERR_ARG   # positions 250..259 need a second table entry
    with pytest.raises(tq4.TQ4Error):
        tq4.tq4_ctx_create([1] * 255 + [0])


def test_inconsistent_device_seq_len_is_recorded():
    ctx = tq4.Context(I.signs(0))
    pool = tq4.Context.new_pool(2)
    table = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    q = torch.zeros(1, 1, 24, 256, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([600], dtype=torch.int32, device="cuda")   # more than the 2-page table holds
    ctx.decode_attention(pool, q, table, seq, 512, SCALE)
    assert ctx.status() == tq4.TQ4_ERR_SEQ
