"""The decode's workspace is scratch: results must not depend on what it held
before (garbage, another call's partials, another context's), and a captured
call must give the same bits on every replay, with eager calls on the same
workspace in between. Every case must equal the oracle within the bf16 tolerance
(fp32 within 1e-4) and the first clean result bit for bit."""
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


@pytest.fixture(scope="module")
def case():
    # three requests, ragged, one of them shorter than a split
    return Case(41, [5000, 700, 12345], 1)


def _args(case, q_bits):
    return (case.pool, _bf16_tensor(q_bits), torch.from_numpy(case.tab).cuda(),
            torch.from_numpy(case.seq_lens).cuda(), int(case.seq_lens.sum()), SCALE)


def _run(ctx, args, ws, out):
    ctx.decode_attention(*args, out=out, workspace=ws)


def test_garbage_workspace_and_repeats(case):
    q_bits = I.queries(41, 0, (3, 1, 24, 256))
    args = _args(case, q_bits)
    ctx = case.ctx
    ws = ctx.decode_workspace(3, 1, int(case.seq_lens.sum()))
    out = torch.empty((3, 1, 24, 256), dtype=torch.bfloat16, device="cuda")
    exp = case.oracle_decode(q_bits)
    first = None
    for fill in (None, 0xFF, 0x00, 0x5A, "random"):
        if fill == "random":
            ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device="cuda"))
        elif fill is not None:
            ws.fill_(fill)
        for _ in range(2):
            _run(ctx, args, ws, out)
            torch.cuda.synchronize()
            assert ctx.status() == tq4.TQ4_OK
            got = out.float().cpu().numpy()
            H.assert_bf16_close(got, exp, f"workspace fill {fill}")
            if first is None:
                first = out.clone()
            assert torch.equal(out, first)


def test_graph_replays_with_eager_calls_between(case):
    q_bits = I.queries(41, 1, (3, 1, 24, 256))
    args = _args(case, q_bits)
    ctx = case.ctx
    ws = ctx.decode_workspace(3, 1, int(case.seq_lens.sum()))
    ref = torch.empty((3, 1, 24, 256), dtype=torch.float32, device="cuda")
    _run(ctx, args, ws, ref)
    torch.cuda.synchronize()
    exp = case.oracle_decode(q_bits)
    assert np.abs(ref.cpu().numpy() - exp).max() <= H.F32_ABS_TOL * max(1.0, np.abs(exp).max())
    out = torch.empty_like(ref)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _run(ctx, args, ws, out)   # warm-up outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            ctx.decode_attention(*args, out=out, workspace=ws, stream=s.cuda_stream)
        for rnd in range(3):
            for _ in range(3):
                out.zero_()
                g.replay()
                torch.cuda.synchronize()
                assert torch.equal(out, ref), f"graph replay, round {rnd}"
            _run(ctx, args, ws, out)   # an eager call with a new tag on the same workspace
            torch.cuda.synchronize()
            assert torch.equal(out, ref)
    assert ctx.status() == tq4.TQ4_OK
    del g


def test_two_contexts_alternate_on_one_workspace(case):
    q_bits = I.queries(41, 2, (3, 1, 24, 256))
    args = _args(case, q_bits)
    other = tq4.Context(case.signs)
    ws = case.ctx.decode_workspace(3, 1, int(case.seq_lens.sum()))
    ref = torch.empty((3, 1, 24, 256), dtype=torch.bfloat16, device="cuda")
    _run(case.ctx, args, ws, ref)
    out = torch.empty_like(ref)
    for i in range(6):
        _run(other if i % 2 == 0 else case.ctx, args, ws, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert other.status() == tq4.TQ4_OK and case.ctx.status() == tq4.TQ4_OK
