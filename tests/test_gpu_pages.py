"""Page tables from the host page pool drive the CUDA path: two requests, the
second restoring a prefix of the first (full pages shared by reference, the
partial page copied on the device) and appending its own positions, then both
decoded in one call, against the fp64 oracle built on the same tables and the
same page copy."""
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
CFG = 21


def test_decode_over_pool_tables_with_restored_prefix():
    signs = I.signs(CFG)
    c, _ = O.codebook()
    ctx = tq4.Context(signs)
    n_pages, max_pages = 12, 6
    pp = tq4.PagePool(n_pages)
    pool = tq4.Context.new_pool(n_pages)
    opool = O.new_pool(n_pages)

    # request A: 1,000 positions (pages 0..3)
    rc, a, _, _ = pp.admit(1000, 64)
    assert rc == tq4.TQ4_OK and pp.grow(a, 1000) == tq4.TQ4_OK
    _, row_a, _ = pp.table(a, max_pages)
    ka, va = I.kv_vectors(CFG, 0, 1000, outlier_frac=0.05)
    ctx.encode_append(pool, torch.tensor(row_a, dtype=torch.int32, device="cuda"), 0,
                      torch.from_numpy(ka).cuda(), torch.from_numpy(va).cuda())
    O.encode_append(opool, np.array(row_a, np.int32), 0, ka, va, signs, c)
    qb = I.queries(CFG, 0, (2, 1, 24, 256))
    qf = I.bf16_bits_to_f32(qb).astype(np.float64)
    exp_a = O.decode_attention(opool, np.array([row_a], np.int32), [1000], qf[:1], SCALE, signs, c)

    # request B restores A's first 700 positions: 2 full pages shared, page 2 copied
    rc, b, cs, cd = pp.admit(900, 64, a, 700)
    assert rc == tq4.TQ4_OK and cs == row_a[2] and cd not in row_a
    pv = pool.view(n_pages, tq4.PAGE_BYTES)
    pv[cd].copy_(pv[cs])
    opv = opool.reshape(n_pages, O.PAGE_BYTES)
    opv[cd] = opv[cs]
    # B prefills 200 positions of its own (700..899), overwriting slots of its copy
    assert pp.grow(b, 900) == tq4.TQ4_OK
    _, row_b, _ = pp.table(b, max_pages)
    assert row_b[:2] == row_a[:2] and row_b[2] == cd
    kb, vb = I.kv_vectors(CFG, 0, 200, first_pos=700, request=1, outlier_frac=0.05)
    ctx.encode_append(pool, torch.tensor(row_b, dtype=torch.int32, device="cuda"), 700,
                      torch.from_numpy(kb).cuda(), torch.from_numpy(vb).cuda())
    O.encode_append(opool, np.array(row_b, np.int32), 700, kb, vb, signs, c)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK

    tables = np.array([row_a, row_b], np.int32)
    seq = np.array([1000, 900], np.int32)
    q = torch.from_numpy(np.ascontiguousarray(qb).view(np.int16)).view(torch.bfloat16).cuda()
    got = ctx.decode_attention(pool, q, torch.from_numpy(tables).cuda(), torch.from_numpy(seq).cuda(),
                               int(seq.sum()), SCALE)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    exp = O.decode_attention(opool, tables, seq, qf, SCALE, signs, c)
    H.assert_bf16_close(got.float().cpu().numpy(), exp, "decode over pool tables")
    # A's output is the one it had before B existed: B wrote only into its own pages
    H.assert_bf16_close(got[:1].float().cpu().numpy(), exp_a, "request A after B's writes")

    # both leave; every page returns at the boundary
    assert pp.finish(a) == tq4.TQ4_OK and pp.finish(b) == tq4.TQ4_OK
    assert pp.step_boundary() == 4 + 2 and pp.free_count() == n_pages
