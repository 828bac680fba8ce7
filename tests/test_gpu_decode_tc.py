"""The tensor-memory decode of 2 to 4 query tokens (tcgen05 MMAs, positions as the
MMA's rows) against the fp64 oracle and against the warp-level mma.sync kernel:
bf16 tolerance on the GPU-encoded pool, 1e-4 in fp32 on the oracle's own pool
bytes, and the two kernels equal to fp32 summation order. Cases cover one tile and
ragged tails, several requests with shared pages, both value-side product sets
(V norms under and over the threshold), scores that keep raising the softmax
reference, the causal limits of each token, and a timeout of the kernel's bounded
waits."""
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
from test_gpu_parity import Case, _bf16_tensor, SCALE  # noqa: E402


def _both_paths(case, q_bits, pool, out_dtype):
    outs = []
    for path in (tq4.DECODE_PATH_TENSOR_MEMORY, tq4.DECODE_PATH_WARP_MMA):
        case.ctx.set_decode_path(path)
        o = case.ctx.decode_attention(pool, _bf16_tensor(q_bits), torch.from_numpy(case.tab).cuda(),
                                      torch.from_numpy(case.seq_lens).cuda(), int(case.seq_lens.sum()), SCALE,
                                      out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert case.ctx.status() == tq4.TQ4_OK
        outs.append(o.float().cpu().numpy().astype(np.float64))
    return outs


@pytest.mark.parametrize("seq_lens,n_q,shared,outliers", [
    ([2], 2, 0, 0.0),                 # inside one tile, token 0 sees one position
    ([128], 2, 0, 0.0),               # exactly one tile
    ([129], 3, 0, 0.05),              # one position into the second tile
    ([300], 2, 0, 0.05),
    ([513, 40], 3, 0, 0.05),          # several requests, a short one
    ([2048, 700], 4, 2, 0.05),        # shared pages
    ([4], 4, 0, 0.0),                 # the shortest four-token history
    ([5000], 4, 0, 0.0),              # no outliers: the value side's lo pass mostly skipped
    ([5000], 4, 0, 0.2),              # many outliers: mostly taken
    ([9000, 4500], 4, 0, 0.05),       # long items
])
def test_tensor_memory_decode_parity(seq_lens, n_q, shared, outliers):
    case = Case(31, seq_lens, n_q, shared_pages=shared, outliers=outliers, chunks=(700,))
    q = I.queries(31, 2, (len(seq_lens), n_q, 24, 256))
    exp = case.oracle_decode(q)
    tm, wm = _both_paths(case, q, case.pool, torch.bfloat16)
    H.assert_bf16_close(tm, exp, f"tensor-memory decode {seq_lens} n_q={n_q}")
    opool = torch.from_numpy(case.opool).cuda()
    tm32, wm32 = _both_paths(case, q, opool, torch.float32)
    scale = max(1.0, np.abs(exp).max())
    assert np.abs(tm32 - exp).max() <= H.F32_ABS_TOL * scale
    assert np.abs(tm32 - wm32).max() <= 1e-5 * scale


def test_tensor_memory_decode_rising_scores():
    """Keys whose scores climb along the history (a query aligned with a key
    direction whose weight grows), so the lazily raised reference is raised in many
    tiles and O is rescaled repeatedly."""
    case = Case(32, [6000], 4, outliers=0.0, chunks=(6000,))
    n = 6000
    k, v = I.kv_vectors(32, 0, n)
    ramp = np.linspace(0.0, 6.0, n, dtype=np.float32)[:, None, None]
    k = (k + ramp * k[:1]).astype(np.float32)          # every key leans further toward key 0
    pool = tq4.Context.new_pool(case.num_pages)
    opool = O.new_pool(case.num_pages)
    case.ctx.encode_append(pool, torch.from_numpy(case.tab[0]).cuda(), 0, torch.from_numpy(k).cuda(),
                           torch.from_numpy(v).cuda())
    O.encode_append(opool, case.tab[0], 0, k, v, case.signs, case.c)
    case.opool = opool
    # queries along key 0's direction, so the scores rise with the ramp
    q = np.repeat(np.repeat(k[:1, :1, :], 24, axis=1)[:, None], 4, axis=1)   # [1, 4, 24, 256]
    q_bits = I.to_bf16_bits(q.astype(np.float32))
    exp = case.oracle_decode(q_bits)
    tm32, wm32 = _both_paths(case, q_bits, torch.from_numpy(opool).cuda(), torch.float32)
    scale = max(1.0, np.abs(exp).max())
    assert np.abs(tm32 - exp).max() <= H.F32_ABS_TOL * scale
    assert np.abs(tm32 - wm32).max() <= 1e-5 * scale


def test_tensor_memory_decode_wait_runs_out_and_context_recovers():
    """The key producers withhold their first chunk's signal: the issuer's bounded
    wait runs out, the kernel records TQ4_ERR_TIMEOUT, drains, frees its tensor
    memory and returns; the context then gives correct results."""
    case = Case(33, [3000], 4, outliers=0.05)
    case.ctx.set_decode_path(tq4.DECODE_PATH_TENSOR_MEMORY)
    q = I.queries(33, 0, (1, 4, 24, 256))
    opool = torch.from_numpy(case.opool).cuda()
    args = (opool, _bf16_tensor(q), torch.from_numpy(case.tab).cuda(), torch.from_numpy(case.seq_lens).cuda(),
            3000, SCALE)
    case.ctx.set_wait_limit(2000, withhold_signal=True)
    case.ctx.decode_attention(*args, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_ERR_TIMEOUT
    case.ctx.set_wait_limit(0)
    out = case.ctx.decode_attention(*args, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert case.ctx.status() == tq4.TQ4_OK
    exp = case.oracle_decode(q)
    assert np.abs(out.cpu().numpy().astype(np.float64) - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())


def test_decode_path_argument_check():
    ctx = tq4.Context(I.signs(0))
    assert tq4.tq4_ctx_set_decode_path(ctx.handle, 2) == tq4.TQ4_ERR_ARG
    assert tq4.tq4_ctx_set_decode_path(ctx.handle, -1) == tq4.TQ4_ERR_ARG
    assert tq4.tq4_ctx_set_decode_path(ctx.handle, tq4.DECODE_PATH_WARP_MMA) == tq4.TQ4_OK
