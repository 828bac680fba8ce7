"""tq4_decode_attention_noalloc: the decode entry point for callers that cannot
allocate device memory (plugin code inside a host program that owns the device
memory budget; serving processes that reserve all memory up front). Its split-K
scratch is the library's fixed device array instead of a caller workspace. It
runs the same kernels with the same plan as the workspace entry point, so its
results must be bit-identical to that entry point's, call after call, and a
smaller call after a larger one must not read the larger call's leftovers."""
import numpy as np
import pytest

from compressed_paged_kv_tq4_b200 import inputs as I

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from compressed_paged_kv_tq4_b200 import tq4  # noqa: E402

SCALE = 1.0 / 16.0


def _problem(ctx, n_q, seq_lens, config=31):
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
    return pool, pool_pages, q, tabs, seq, int(sum(seq_lens))


def _noalloc(ctx, prob, n_q, out_dtype):
    pool, pool_pages, q, tabs, seq, total = prob
    out = torch.empty(q.shape, dtype=out_dtype, device="cuda")
    od = tq4.DTYPE_F32 if out_dtype == torch.float32 else tq4.DTYPE_BF16
    rc = tq4.tq4_decode_attention_noalloc(ctx.handle, pool, pool_pages, q, tabs, tabs.shape[1], seq,
                                          seq.numel(), n_q, total, SCALE, out, od)
    assert rc == tq4.TQ4_OK, tq4.tq4_status_string(rc)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    return out


def _reference(ctx, prob, out_dtype):
    pool, _, q, tabs, seq, total = prob
    out = ctx.decode_attention(pool, q, tabs, seq, total, SCALE, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    return out


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_noalloc_equals_workspace_entry_point_large_call_then_small_call(out_dtype):
    """A large call (4 query tokens, many splits) fills much of the fixed array; the
    smaller one-token call that follows must still equal the workspace entry point
    bit for bit, and so must a repeat of each."""
    ctx = tq4.Context(I.signs(31))
    big = _problem(ctx, 4, [9000, 2048, 333])
    small = _problem(ctx, 1, [700, 1300])
    ref_big, ref_small = _reference(ctx, big, out_dtype), _reference(ctx, small, out_dtype)
    for prob, n_q, ref in ((big, 4, ref_big), (small, 1, ref_small), (big, 4, ref_big), (small, 1, ref_small)):
        got = _noalloc(ctx, prob, n_q, out_dtype)
        assert torch.equal(got, ref)


def _plan_bytes(ctx, n_req, n_q, seq):
    return tq4.tq4_decode_workspace_bytes(ctx.handle, n_req, n_q, n_req * seq)


@pytest.mark.parametrize("n_q", [1, 4])
def test_noalloc_limit_boundary(n_q):
    """The largest batch of 16-position requests whose workspace fits the fixed array
    runs (and equals the workspace entry point); one request more is rejected with
    TQ4_ERR_WORKSPACE before anything is launched."""
    ctx = tq4.Context(I.signs(31))
    seq = 16
    n = 1
    while _plan_bytes(ctx, n + 1, n_q, seq) <= tq4.NOALLOC_SCRATCH_BYTES:
        n += 1
    assert _plan_bytes(ctx, n, n_q, seq) <= tq4.NOALLOC_SCRATCH_BYTES < _plan_bytes(ctx, n + 1, n_q, seq)
    # rejected on the host: nothing is launched, so the (dummy) pointers are never read
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = tq4.tq4_decode_attention_noalloc(ctx.handle, dummy, 1, dummy, dummy, 16, dummy, n + 1, n_q,
                                          (n + 1) * seq, SCALE, dummy, tq4.DTYPE_BF16)
    assert rc == tq4.TQ4_ERR_WORKSPACE
    assert ctx.status() == tq4.TQ4_OK
    prob = _problem(ctx, n_q, [seq] * n)
    assert torch.equal(_noalloc(ctx, prob, n_q, torch.bfloat16), _reference(ctx, prob, torch.bfloat16))
