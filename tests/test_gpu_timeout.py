"""Bounded device waits that run out, without a GPU fault.

The context's test hook (tq4_ctx_set_wait_limit) lowers the poll limit of the
bounded waits and withholds one producer signal, so that a wait is sure to run
out: the one-token decode kernel does not issue the copy of each warp's first
tile; the prefill kernel's softmax warps do not tell the tensor-core issuer that
one tile's P is ready, after some tensor-core operations of the CTA pair have
been issued. The kernel must record TQ4_ERR_TIMEOUT, drain what it issued, free
its tensor memory and return; the same context must then give correct results."""
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
POLLS = 2000   # a few hundred microseconds of polling at most


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _pool(config, n, outliers=0.0):
    signs = I.signs(config)
    npg = (n + 255) // 256
    table = I.page_table_scattered(config, npg, npg + 1)
    k, v = I.kv_vectors(config, 0, n, outlier_frac=outliers)
    opool = O.new_pool(npg + 1)
    O.encode_append(opool, table, 0, k, v, signs, O.codebook()[0])
    return signs, table, opool


def test_decode_wait_runs_out_and_context_recovers():
    signs, table, opool = _pool(11, 3000)
    ctx = tq4.Context(signs)
    pool = torch.from_numpy(opool).cuda()
    tab = torch.from_numpy(table[None]).cuda()
    seq = torch.tensor([3000], dtype=torch.int32, device="cuda")
    qb = I.queries(11, 0, (1, 1, 24, 256))
    q = _bf16_tensor(qb)
    ctx.set_wait_limit(POLLS, withhold_signal=True)
    ctx.decode_attention(pool, q, tab, seq, 3000, SCALE, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_ERR_TIMEOUT
    ctx.set_wait_limit(0)   # default limit, no withheld signal
    out = ctx.decode_attention(pool, q, tab, seq, 3000, SCALE, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    exp = O.decode_attention(opool, table[None], [3000], I.bf16_bits_to_f32(qb), SCALE, signs, O.codebook()[0])
    err = np.abs(out.cpu().numpy().astype(np.float64) - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())


@pytest.mark.parametrize("prefix_len,n_tok", [(700, 100), (0, 3)])
def test_prefill_wait_runs_out_drains_and_context_recovers(prefix_len, n_tok):
    signs, table, opool = _pool(12, max(prefix_len, 1))
    ctx = tq4.Context(signs)
    pool = torch.from_numpy(opool).cuda()
    tt = torch.from_numpy(table).cuda()
    qb = I.queries(12, 0, (n_tok, 24, 256))
    kb, vb = I.chunk_kv(12, 0, n_tok)
    args = (pool, tt, prefix_len, _bf16_tensor(qb), _bf16_tensor(kb), _bf16_tensor(vb), SCALE)
    ctx.set_wait_limit(POLLS, withhold_signal=True)
    ctx.prefill_attention(*args, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_ERR_TIMEOUT
    ctx.set_wait_limit(0)
    out = ctx.prefill_attention(*args, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctx.status() == tq4.TQ4_OK
    exp = O.prefill_attention(opool, table, prefix_len, I.bf16_bits_to_f32(qb), I.bf16_bits_to_f32(kb),
                              I.bf16_bits_to_f32(vb), SCALE, signs, O.codebook()[0])
    err = np.abs(out.cpu().numpy().astype(np.float64) - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())
