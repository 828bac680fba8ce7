"""GPU parity of the uniform INT8 comparison arm against its fp64 oracle
(oracle/int8_oracle.py), through the C ABI: the encode is bit-exact (its
divisions and rounding are done in fp64, as the oracle's are); decode attention
meets the bf16 tolerance on the GPU-encoded pool and 1e-4 (fp32 output) on the
oracle's own pool bytes, for 1 to 4 query tokens, ragged lengths, shared pages
and a 32,768-position history."""
import numpy as np
import pytest

from compressed_paged_kv_tq4_b200 import inputs as I
from oracle import int8_oracle as O8
import _helpers as H

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from compressed_paged_kv_tq4_b200 import tq4  # noqa: E402

SCALE = 1.0 / 16.0


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_int8_encode_bit_exact(dtype):
    ctx = tq4.Context(I.signs(0))
    table = I.page_table_scattered(21, 5, 7)
    k, v = I.kv_vectors(21, 0, 1200, outlier_frac=0.05)
    k[17] = 0.0                                   # a zero vector
    if dtype == "bf16":
        kb, vb = I.to_bf16_bits(k), I.to_bf16_bits(v)
        k, v = I.bf16_bits_to_f32(kb), I.bf16_bits_to_f32(vb)
        kt, vt = _bf16_tensor(kb), _bf16_tensor(vb)
    else:
        kt, vt = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    pool = tq4.Context.new_int8_pool(7)
    tt = torch.from_numpy(table).cuda()
    for a, e in ((0, 333), (333, 1000), (1000, 1200)):   # appends that start mid-page
        ctx.int8_encode_append(pool, tt, a, kt[a:e], vt[a:e])
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    opool = O8.new_pool(7)
    O8.encode_append(opool, table, 0, k, v)
    pages = np.unique(table[:5])
    got = pool.cpu().numpy().reshape(7, -1)[pages]
    exp = opool.reshape(7, -1)[pages]
    assert np.array_equal(got, exp)


class Int8Case:
    def __init__(self, config, seq_lens, n_q, shared_pages=0, outliers=0.05):
        self.ctx = tq4.Context(I.signs(config))
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
        self.tab, self.num_pages, self.n_q = tab, total, n_q
        self.seq = np.array(seq_lens, np.int32)
        self.pool = tq4.Context.new_int8_pool(total)
        self.opool = O8.new_pool(total)
        for r, s in enumerate(seq_lens):
            first = shared_pages * 256 if r > 0 else 0
            k, v = I.kv_vectors(config, 0, s - first, first_pos=first, request=r, outlier_frac=outliers)
            self.ctx.int8_encode_append(self.pool, torch.from_numpy(tab[r]).cuda(), first,
                                        torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            O8.encode_append(self.opool, tab[r], first, k, v)
        torch.cuda.synchronize()
        assert self.ctx.status() == tq4.TQ4_OK

    def decode(self, qb, pool, out_dtype):
        out = self.ctx.int8_decode_attention(pool, _bf16_tensor(qb), torch.from_numpy(self.tab).cuda(),
                                             torch.from_numpy(self.seq).cuda(), int(self.seq.sum()), SCALE,
                                             out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert self.ctx.status() == tq4.TQ4_OK
        return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("seq_lens,n_q,shared", [
    ([1], 1, 0), ([255], 1, 0), ([257], 1, 0), ([1000, 63, 2047], 1, 0), ([300], 2, 0),
    ([513, 40], 3, 0), ([2048, 700], 4, 2), ([4], 4, 0), ([5000], 4, 0), ([20000], 1, 0),
])
def test_int8_decode_parity(seq_lens, n_q, shared):
    case = Int8Case(23, seq_lens, n_q, shared_pages=shared)
    qb = I.queries(23, 1, (len(seq_lens), n_q, 24, 256))
    exp = O8.decode_attention(case.opool, case.tab, case.seq, I.bf16_bits_to_f32(qb), SCALE)
    H.assert_bf16_close(case.decode(qb, case.pool, torch.bfloat16), exp, f"int8 decode {seq_lens} n_q={n_q}")
    got32 = case.decode(qb, torch.from_numpy(case.opool).cuda(), torch.float32)
    err = np.abs(got32 - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), err


def test_int8_decode_32k_history():
    """The decode_32k shape (one request, 32,768 positions, one query token) on the INT8 arm."""
    case = Int8Case(24, [32768], 1, outliers=0.0)
    qb = I.queries(24, 0, (1, 1, 24, 256))
    exp = O8.decode_attention(case.opool, case.tab, case.seq, I.bf16_bits_to_f32(qb), SCALE)
    got32 = case.decode(qb, torch.from_numpy(case.opool).cuda(), torch.float32)
    assert np.abs(got32 - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())
    H.assert_bf16_close(case.decode(qb, case.pool, torch.bfloat16), exp, "int8 decode 32k")
