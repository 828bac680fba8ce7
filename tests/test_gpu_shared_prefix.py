"""Shared-prefix dedup (tq4_decode_attention_shared): requests whose tables hold
the same leading page ids are grouped, and each group's shared positions are
loaded and expanded once for all members' query rows. Checked against the fp64
oracle (bf16 tolerance on the GPU-encoded pool, 1e-4 in fp32 on the oracle's own
pool bytes) and against the ungrouped decode, over one to four query tokens,
groups cut by the row cap, requests outside any group, the append, and the
argument checks of the group description."""
import numpy as np
import pytest

from compressed_paged_kv_tq4_b200 import inputs as I
import _helpers as H

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from compressed_paged_kv_tq4_b200 import tq4  # noqa: E402
from test_gpu_parity import Case, _bf16_tensor, SCALE  # noqa: E402


def _shared(case, q_bits, leader, pages, out_dtype, pool=None):
    out = case.ctx.decode_attention_shared(
        case.pool if pool is None else pool, _bf16_tensor(q_bits), torch.from_numpy(case.tab).cuda(),
        torch.from_numpy(case.seq_lens).cuda(), int(case.seq_lens.sum()), SCALE, leader, pages,
        out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_OK
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("seq_lens,n_q,shared,leader", [
    ([3000, 2500, 4000], 1, 8, [0, 0, 0]),            # one group of three, one token
    ([3000, 700, 2900, 5000], 2, 2, [0, 0, 0, 3]),    # a group of three; request 3 alone
    ([9000, 4500], 4, 16, [0, 0]),                    # the verify shape: two four-token requests
    ([2600, 2600, 2700], 4, 8, [0, 0, 0]),            # three four-token members: cut to 2 + 1
    ([1100, 1300, 1500, 1700, 1900, 2100, 2300, 2500, 2700], 1, 4, [0] * 9),   # nine: cut to 8 + 1
])
def test_shared_prefix_parity(seq_lens, n_q, shared, leader):
    case = Case(51, seq_lens, n_q, shared_pages=shared, outliers=0.05, chunks=(777,))
    pages = [shared if leader[r] == 0 else 0 for r in range(len(seq_lens))]
    q_bits = I.queries(51, 0, (len(seq_lens), n_q, 24, 256))
    exp = case.oracle_decode(q_bits)
    got = _shared(case, q_bits, leader, pages, torch.bfloat16)
    H.assert_bf16_close(got, exp, f"shared prefix {seq_lens} n_q={n_q}")
    got32 = _shared(case, q_bits, leader, pages, torch.float32, pool=torch.from_numpy(case.opool).cuda())
    err = np.abs(got32 - exp).max()
    assert err <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max()), err
    # the ungrouped decode computes the same values (fp32, up to summation order)
    plain = case.decode_oracle_pool(q_bits, torch.float32)
    assert np.abs(got32 - plain).max() <= 1e-5 * max(1.0, np.abs(plain).max())


def test_shared_prefix_with_append():
    """k_new / v_new given: the step's tokens are appended (tail encode), then the
    grouped decode runs; equal to the ungrouped append + decode within fp32 order."""
    n_q = 4
    case = Case(52, [6000, 3000], n_q, shared_pages=8)
    k_new, v_new = [], []
    for r, s in enumerate(case.seq_lens):
        k, v = I.kv_vectors(52, 1, n_q, first_pos=int(s), request=r)
        k_new.append(k)
        v_new.append(v)
    kt = torch.from_numpy(np.stack(k_new)).cuda()
    vt = torch.from_numpy(np.stack(v_new)).cuda()
    seq = case.seq_lens + n_q
    q_bits = I.queries(52, 0, (2, n_q, 24, 256))
    tab = torch.from_numpy(case.tab).cuda()
    pool2 = case.pool.clone()
    a = case.ctx.decode_attention_shared(case.pool, _bf16_tensor(q_bits), tab, torch.from_numpy(seq).cuda(),
                                         int(seq.sum()), SCALE, [0, 0], [8, 8], k_new=kt, v_new=vt,
                                         out_dtype=torch.float32)
    b = case.ctx.decode_append_attention(pool2, kt, vt, _bf16_tensor(q_bits), tab, torch.from_numpy(seq).cuda(),
                                         int(seq.sum()), SCALE, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_OK
    assert torch.equal(case.pool, pool2)   # the same bytes appended
    assert (a - b).abs().max().item() <= 1e-5 * max(1.0, b.abs().max().item())


def test_shared_prefix_argument_checks():
    case = Case(53, [600, 600], 1, shared_pages=2)
    q = _bf16_tensor(I.queries(53, 0, (2, 1, 24, 256)))
    tab = torch.from_numpy(case.tab).cuda()
    seq = torch.from_numpy(case.seq_lens).cuda()
    max_pages = tab.shape[1]
    for leader, pages in (([0, 2], [2, 2]),      # leader out of range
                          ([1, 0], [2, 2]),      # leaders that are not their own leaders
                          ([0, 0], [2, 1]),      # unequal page counts in a group
                          ([0, 0], [-1, -1]),    # negative
                          ([0, 0], [max_pages + 1] * 2)):
        assert tq4.tq4_decode_shared_workspace_bytes(case.ctx.handle, 2, 1, 1200, max_pages, leader, pages) == 0
        ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        out = torch.empty(2, 1, 24, 256, dtype=torch.bfloat16, device="cuda")
        rc = tq4.tq4_decode_attention_shared(case.ctx.handle, case.pool, case.num_pages, None, None, tq4.DTYPE_F32,
                                             q, tab, max_pages, seq, 2, 1, 1200, leader, pages, SCALE, out,
                                             tq4.DTYPE_BF16, ws, ws.numel())
        assert rc == tq4.TQ4_ERR_ARG, (leader, pages, rc)
    assert case.ctx.status() == tq4.TQ4_OK
