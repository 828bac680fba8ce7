"""tq4_decode_attention_noalloc: the decode entry point for callers that cannot
allocate device memory (plugin code inside a host program that owns the device
memory budget; serving processes that reserve all memory up front). Its split-K
scratch is the library's fixed device array instead of a caller workspace; its
results must match the workspace entry point's, call after call."""
import numpy as np
import pytest

from compressed_paged_kv_tq4_b200 import inputs as I
import _helpers as H

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from compressed_paged_kv_tq4_b200 import tq4  # noqa: E402

SCALE = 1.0 / 16.0


def _problem(n_q, seq_lens, config=31):
    signs = I.signs(config)
    ctx = tq4.Context(signs)
    npg = [(s + 255) // 256 for s in seq_lens]
    pool_pages = sum(npg) + 2
    ids = I.page_table_scattered(config, sum(npg), pool_pages)
    tab = np.full((len(seq_lens), max(npg)), -1, np.int32)
    off = 0
    for r, n in enumerate(npg):
        tab[r, :n] = ids[off:off + n]
        off += n
    pool = tq4.Context.new_pool(pool_pages)
    tabs = torch.from_numpy(tab).cuda()
    for r, s in enumerate(seq_lens):
        k, v = I.kv_vectors(config, 0, s, request=r, outlier_frac=0.05)
        ctx.encode_append(pool, tabs[r], 0, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    qb = I.queries(config, 0, (len(seq_lens), n_q, 24, 256))
    q = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).cuda()
    seq = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    return ctx, pool, pool_pages, q, tabs, seq, int(sum(seq_lens))


@pytest.mark.parametrize("n_q,seq_lens", [(1, [700, 1300]), (4, [2048, 333])])
def test_noalloc_matches_workspace_entry_point_twice(n_q, seq_lens):
    ctx, pool, pool_pages, q, tabs, seq, total = _problem(n_q, seq_lens)
    ref = ctx.decode_attention(pool, q, tabs, seq, total, SCALE)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    for _ in range(2):   # the fixed scratch keeps the previous call's contents
        out = torch.empty_like(ref)
        rc = tq4.tq4_decode_attention_noalloc(ctx.handle, pool, pool_pages, q, tabs, tabs.shape[1], seq,
                                              len(seq_lens), n_q, total, SCALE, out, tq4.DTYPE_BF16)
        assert rc == tq4.TQ4_OK, tq4.tq4_status_string(rc)
        torch.cuda.synchronize()
        assert ctx.status() == tq4.TQ4_OK
        H.assert_bf16_close(out.float().cpu().numpy(), ref.float().cpu().numpy(), "no-alloc vs workspace")


def test_noalloc_rejects_problems_beyond_its_scratch():
    ctx = tq4.Context(I.signs(31))
    n_req, n_q = 300, 4
    total = n_req * 4096
    need = tq4.tq4_decode_workspace_bytes(ctx.handle, n_req, n_q, total)
    assert need > tq4.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = tq4.tq4_decode_attention_noalloc(ctx.handle, dummy, 1, dummy, dummy, 16, dummy, n_req, n_q, total,
                                          SCALE, dummy, tq4.DTYPE_BF16)
    assert rc == tq4.TQ4_ERR_WORKSPACE
