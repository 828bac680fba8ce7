"""Host page pool (include/tq4_pages.h) against the oracle model (oracle/page_pool.py).

The oracle model is pinned first by what the page fixes independently of it: the
admission formula on the page's own workload numbers, a worked example traced by
hand, and invariants (reference counts equal table membership, no page is freed
before a boundary, capacity is conserved). The library is then compared with the
model result by result on seeded random operation sequences. No GPU is used.
"""
import random
import time

import numpy as np
import pytest

from oracle import page_pool as M

tq4 = pytest.importorskip("compressed_paged_kv_tq4_b200.tq4")

POOL_229K = 229_376 // 256   # the page's capacity runs use a 229,376-position pool


# ---------------------------------------------------------------- pins of the model
def test_reservation_formula_on_the_pages_workloads():
    # [STATE]: ceil((prompt + min(output budget, 8192)) / 256)
    assert POOL_229K == 896
    # single capacity run: 196,608 prompt + 16,384 output -> (196,608 + 8,192) / 256
    assert M.reservation(196_608, 16_384) == 800
    # two concurrent requests of 96K + 16K each
    assert M.reservation(98_304, 16_384) == 416
    # the output term saturates at 8,192; below it, it counts in full
    assert M.reservation(0, 100_000) == M.reservation(0, 8192) == 32
    assert M.reservation(1, 0) == 1 and M.reservation(256, 0) == 1 and M.reservation(257, 0) == 2
    assert M.reservation(-1, 0) == -1 and M.reservation(0, -1) == -1
    for prompt, out in ((196_608, 16_384), (98_304, 16_384), (0, 100_000), (1, 0), (257, 0), (5, 7)):
        assert tq4.tq4_pages_reservation(prompt, out) == M.reservation(prompt, out)
    assert tq4.tq4_pages_reservation(-1, 0) == -1


@pytest.mark.parametrize("impl", ["model", "library"])
def test_capacity_runs_of_the_page(impl):
    pool = M.PagePoolModel(POOL_229K) if impl == "model" else tq4.PagePool(POOL_229K)
    # one 196,608 + 16,384 request fits with 96 page equivalents to spare
    rc, a, _, _ = pool.admit(196_608, 16_384)
    assert rc == 0 and pool.available() == 96
    assert pool.finish(a) == 0 and pool.step_boundary() == 0 and pool.available() == 896
    # two 96K + 16K requests fit together (832 of 896); a third does not
    rc1, r1, _, _ = pool.admit(98_304, 16_384)
    rc2, r2, _, _ = pool.admit(98_304, 16_384)
    assert (rc1, rc2) == (0, 0) and pool.available() == 64
    assert pool.admit(98_304, 16_384)[0] == M.ERR_NO_PAGES
    # prefilling the prompts maps 384 pages each, inside the reservations
    assert pool.grow(r1, 98_304) == 0 and pool.grow(r2, 98_304) == 0
    assert pool.free_count() == 896 - 768 and pool.available() == 64


@pytest.mark.parametrize("impl", ["model", "library"])
def test_prefix_restore_of_the_page(impl):
    # [REUSE]: a request restores 16,383 cached positions and prefills one new token
    pool = M.PagePoolModel(POOL_229K) if impl == "model" else tq4.PagePool(POOL_229K)
    rc, a, _, _ = pool.admit(16_383, 64)
    assert rc == 0 and pool.grow(a, 16_383) == 0          # 64 pages, the last one 255 positions full
    rc, b, cs, cd = pool.admit(16_384, 64, a, 16_383)
    assert rc == 0
    ok, ta, la = pool.table(a, 64)
    ok2, tb, lb = pool.table(b, 64)
    assert ok == ok2 == 0 and la == lb == 16_383
    assert tb[:63] == ta[:63]                              # 63 full pages shared by reference
    assert cs == ta[63] and cd == tb[63] and cd not in ta  # the partial page is a private copy
    assert all(pool.refcount(p) == 2 for p in ta[:63]) and pool.refcount(ta[63]) == 1
    assert pool.refcount(cd) == 1
    # the new token is position 16,383: slot 255 of the copied page, no new page
    free_before = pool.free_count()
    assert pool.grow(b, 16_384) == 0 and pool.free_count() == free_before
    # reservation of b: ceil((16,384 + 64) / 256) = 65, less 63 shared pages = 2, one used by the copy
    assert pool.available() == POOL_229K - 64 - 1 - 1 - (M.reservation(16_383, 64) - 64)


@pytest.mark.parametrize("impl", ["model", "library"])
def test_worked_example_by_hand(impl):
    """Six pages, traced by hand from the rules in the model's header."""
    pool = M.PagePoolModel(6) if impl == "model" else tq4.PagePool(6)
    # A: prompt 300, output 100 -> reserve ceil(400 / 256) = 2
    assert pool.admit(300, 100)[:2] == (0, 0)
    assert pool.available() == 4 and pool.free_count() == 6
    assert pool.grow(0, 300) == 0                          # pages 0, 1 (front of the free list)
    assert pool.table(0, 3) == (0, [0, 1, -1], 300)
    assert pool.free_list() == [2, 3, 4, 5] and pool.available() == 4
    # A grows past its reservation (surplus output): page 2 from unreserved capacity
    assert pool.grow(0, 600) == 0 and pool.table(0, 3) == (0, [0, 1, 2], 600)
    assert pool.available() == 3
    # B restores A's first 260 positions: page 0 shared, page 1 copied into page 3
    # reserve = ceil((270 + 10) / 256) - 1 = 1, used by the copy
    assert pool.admit(270, 10, 0, 260) == (0, 1, 1, 3)
    assert pool.table(1, 3) == (0, [0, 3, -1], 260)
    assert [pool.refcount(p) for p in range(6)] == [2, 1, 1, 1, 0, 0]
    assert pool.available() == 2
    # C wants 3 page equivalents: only 2 available
    assert pool.admit(700, 0)[0] == M.ERR_NO_PAGES
    # A leaves: nothing is freed before the boundary
    assert pool.finish(0) == 0
    assert pool.free_list() == [4, 5] and pool.refcount(0) == 2
    assert pool.grow(0, 700) == M.ERR_ARG                  # a leaving request cannot grow
    assert pool.step_boundary() == 2                       # pages 1 and 2 reach zero; page 0 is B's
    assert pool.free_list() == [4, 5, 1, 2] and [pool.refcount(p) for p in range(6)] == [1, 0, 0, 1, 0, 0]
    assert pool.table(0, 3)[0] == M.ERR_ARG                # A is forgotten
    # now C fits: reserve 3 of 4 available
    assert pool.admit(700, 0)[:2] == (0, 2) and pool.available() == 1
    assert pool.grow(2, 700) == 0 and pool.table(2, 3) == (0, [4, 5, 1], 700)
    # B and C leave in one step: page 0 (B's last reference), 3, 4, 5, 1 freed, in id order
    assert pool.finish(1) == 0 and pool.finish(2) == 0
    assert pool.step_boundary() == 5
    assert pool.free_list() == [2, 0, 1, 3, 4, 5] and pool.available() == 6


@pytest.mark.parametrize("impl", ["model", "library"])
def test_argument_errors_change_nothing(impl):
    pool = M.PagePoolModel(4) if impl == "model" else tq4.PagePool(4)
    assert pool.admit(-1, 0)[0] == M.ERR_ARG
    assert pool.admit(10, -1)[0] == M.ERR_ARG
    assert pool.admit(10, 0, -1, 5)[0] == M.ERR_ARG        # a prefix without a source
    assert pool.admit(10, 0, 7, 5)[0] == M.ERR_ARG         # unknown source
    assert pool.admit(300, 0)[:2] == (0, 0) and pool.grow(0, 300) == 0
    assert pool.admit(10, 0, 0, 20)[0] == M.ERR_ARG        # prefix longer than the prompt
    assert pool.admit(400, 0, 0, 301)[0] == M.ERR_ARG      # prefix longer than the source
    assert pool.admit(400, 0, 0, 0)[0] == M.ERR_ARG        # empty prefix with a source
    assert pool.grow(0, 299) == M.ERR_ARG                  # never shrinks
    assert pool.grow(5, 10) == M.ERR_ARG and pool.finish(5) == M.ERR_ARG
    assert pool.admit(2000, 0)[0] == M.ERR_NO_PAGES
    assert pool.grow(0, 5000) == M.ERR_NO_PAGES            # all or nothing
    assert pool.table(0, 4) == (0, [0, 1, -1, -1], 300)
    assert pool.table(0, 1)[0] == M.ERR_ARG                # row does not fit
    assert pool.free_list() == [2, 3] and pool.available() == 2
    assert pool.refcount(4) == M.ERR_ARG and pool.refcount(-1) == M.ERR_ARG


# ---------------------------------------------------------------- random sequences
def _random_ops(seed, n_ops, num_pages):
    """A seeded operation sequence (the same list drives the model and the library)."""
    rng = random.Random(seed)
    ops, live_guess = [], 0
    for _ in range(n_ops):
        x = rng.random()
        if x < 0.25:
            prompt = rng.choice([0, 1, 255, 256, 257, rng.randrange(0, 6 * 256)])
            out = rng.choice([0, 1, 300, rng.randrange(0, 3000)])
            if rng.random() < 0.4:
                ops.append(("admit_restore", prompt, out, rng.randrange(0, max(live_guess, 1) + 2),
                            rng.randrange(0, 5 * 256)))
            else:
                ops.append(("admit", prompt, out))
            live_guess += 1
        elif x < 0.65:
            ops.append(("grow", rng.randrange(0, live_guess + 2), rng.randrange(0, 8 * 256)))
        elif x < 0.8:
            ops.append(("finish", rng.randrange(0, live_guess + 2)))
        else:
            ops.append(("boundary",))
    return ops


def _apply(pool, op):
    kind = op[0]
    if kind == "admit":
        return pool.admit(op[1], op[2])
    if kind == "admit_restore":
        return pool.admit(max(op[1], op[4]), op[2], op[3], op[4])
    if kind == "grow":
        return pool.grow(op[1], op[2])
    if kind == "finish":
        return pool.finish(op[1])
    return pool.step_boundary()


def _check_invariants(model):
    held = {}
    for r in model.reqs.values():
        assert len(r["pages"]) == -(-r["len"] // M.PAGE)
        for p in r["pages"]:
            held[p] = held.get(p, 0) + 1
    for p in range(model.num_pages):
        assert model.refs[p] == held.get(p, 0)            # counts equal table membership
    assert set(model.free) == {p for p in range(model.num_pages) if held.get(p, 0) == 0}
    assert len(model.free) == len(set(model.free))
    assert model.available() >= 0


@pytest.mark.parametrize("seed,num_pages", [(1, 8), (2, 16), (3, 40), (4, 5)])
def test_library_matches_model_on_random_sequences(seed, num_pages):
    model, lib = M.PagePoolModel(num_pages), tq4.PagePool(num_pages)
    held_before = set()
    for op in _random_ops(seed, 600, num_pages):
        got, exp = _apply(lib, op), _apply(model, op)
        assert got == exp, (op, got, exp)
        _check_invariants(model)
        held_now = {p for p in range(num_pages) if model.refs[p] > 0}
        if op[0] != "boundary":                              # pages are only freed at a boundary
            assert held_before <= held_now
        held_before = held_now
        assert lib.free_list() == model.free_list()
        assert lib.available() == model.available()
        assert [lib.refcount(p) for p in range(num_pages)] == model.refs
        for rid in list(model.reqs)[-3:]:
            assert lib.table(rid, num_pages) == model.table(rid, num_pages)


def test_host_throughput():
    """Time a mixed sequence on the library and on the model (reported, not asserted)."""
    ops = _random_ops(9, 20_000, 896)
    out = {}
    for name, pool in (("library", tq4.PagePool(896)), ("model", M.PagePoolModel(896))):
        t0 = time.perf_counter()
        for op in ops:
            _apply(pool, op)
        out[name] = len(ops) / (time.perf_counter() - t0)
    print(f"page pool ops/s through the Python binding: library {out['library']:.3g}, model {out['model']:.3g}")
    assert np.isfinite(out["library"]) and out["library"] > 0


def test_concurrent_callers_keep_the_invariants():
    """Four threads admit, grow and finish their own requests on one pool; the lock
    keeps every page either free or referenced exactly as often as tables hold it."""
    import threading

    pool = tq4.PagePool(64)
    errors = []

    def worker(seed):
        rng = random.Random(seed)
        try:
            for _ in range(300):
                rc, req, _, _ = pool.admit(rng.randrange(1, 700), rng.randrange(0, 300))
                if rc != 0:
                    continue
                for _ in range(rng.randrange(1, 4)):
                    pool.grow(req, rng.randrange(0, 900))
                assert pool.finish(req) == 0
                if rng.random() < 0.5:
                    pool.step_boundary()
        except Exception as e:   # reported below; a thread cannot fail the test directly
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(s,)) for s in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    pool.step_boundary()
    assert pool.free_count() == 64 and pool.available() == 64
    assert sorted(pool.free_list()) == list(range(64))
    assert all(pool.refcount(p) == 0 for p in range(64))
