#!/usr/bin/env python
"""Benchmark of the TQ4 paged-KV attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: for every layer,
tq4_decode_append_attention (the step's new K/V positions appended, then decode
attention over the whole history; with one query token the append runs inside
the decode kernel) for decode workloads, or tq4_prefill_attention followed by
tq4_encode_append of the chunk (prefill workload). The step's launches are captured once in a CUDA
graph through the public C ABI and replayed; the timed region is exactly K
replays between CUDA events, after W warm-up replays.

Prints one JSON line. Multi-GPU runs (torchrun) are independent replicas: the
path has no exchange step, every rank runs the same workload on its own GPU
and the value is the units of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressed_paged_kv_tq4_b200 import inputs as I  # noqa: E402

METRIC = "TQ4 fused attention KV positions/s & HBM GB/s (% of roofline) at 32K–229K ctx"
UNIT = "KV positions/s"
SCALE = 1.0 / 16.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode_32k", choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch without a CUDA graph (profiling)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling only)")
    ap.add_argument("--profile", action="store_true",
                    help="eager steps only: no roofline replay, e2e or CPU leg (for ncu captures)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


WORKLOAD_DESC = {
    "decode_32k": "16 layers x 32,768 TQ4 positions, 1 request, 1 bf16 query token, 24 Q / 4 KV heads x 256",
    "decode_213k_outliers": "16 layers x 212,992 TQ4 positions (5% x8 outliers), 1 request, 1 query token",
    "verify_2req_229k": "2 requests (163,840 + 65,536 positions, 64 shared pages), 4 causal query tokens each, "
                        "16 layers",
    "prefill_2k_on_32k": "2,048 causal bf16 query tokens on a 32,768-position TQ4 prefix + the chunk, 16 layers",
    "single_layer_2k": "1 layer, 2,048 TQ4 positions, 1 query token",
}


def workload_config(name, world):
    """The `config` object of the JSON line (the same for both arms)."""
    w = I.WORKLOADS[name]
    return {"workload": f"{name}: {WORKLOAD_DESC[name]}", "append_per_layer": w.append_per_step,
            "pool_pages": w.pool_pages, "page_positions": 256,
            "l2": "inputs larger than L2: packed KV read per step is "
                  f"{w.layers * sum(w.seq_lens) * 1040 / 1e6:.0f} MB vs 126 MB L2",
            "parallelism": f"replicas x{world}"}


# ---------------------------------------------------------------------------- measured DRAM traffic
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture
# (summarised under profiles/), per unit of work. A figure counts only while the
# kernel's source file hashes to the value it had when the counters were taken.
MEASURED_TRAFFIC = {
    # decode_q1_kernel, decode_32k capture (append fused): 34,172,160 B read + 77,312 B
    # written for 32,768 positions; its traffic grows with the positions it streams
    "decode_q1": ("tq4_decode_q1.cuh", "a1aa9c992fe1114efe87749225ea10ca9eca128a3d97914e4c08bafae57d9706",
                  (34_172_160 + 77_312) / 32_768),
    # decode_splitk_kernel<3>, verify_2req_229k capture: 221,675,264 B read + 3,709,696 B
    # written for 229,376 positions (the 64 shared pages partly hit in L2: this workload only)
    "decode_splitk": ("tq4_decode.cuh", "d27dcffa6032aeb25c0c742e6ca77347597bf628fd34c9a1f3d0b6a41afc0340",
                      (221_675_264 + 3_709_696) / 229_376),
    # prefill_tc_kernel, prefill_2k_on_32k capture: one launch
    "prefill_tc": ("tq4_prefill_tc.cuh", "f290435adb0de7f5ccb086652cf386f89fbab4a08afeb143fa73615e1aa92529",
                   93_480_960 + 9_271_552),
}


def measured_traffic(key, units):
    """Bytes per launch for ``units`` units of work, or None if the kernel changed since the capture."""
    if key not in MEASURED_TRAFFIC:
        return None
    import hashlib
    fname, digest, per_unit = MEASURED_TRAFFIC[key]
    path = os.path.join(ROOT, "compressed_paged_kv_tq4_b200", "csrc", fname)
    try:
        with open(path, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None
    except OSError:
        return None
    return per_unit * units


# ---------------------------------------------------------------------------- replicas (host side)
def max_over_ranks(ms, dist, device):
    """Step time of the whole job: the slowest rank's (every rank calls this, in the same order)."""
    if dist is None:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_step, world, ms):
    """Whole-job throughput: units processed by all ranks over the slowest rank's step time."""
    return units_per_step * world / (ms * 1e-3)


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                break
            time.sleep(0.0005)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------- host data
def gen_kv_parallel(config, layer, n, first_pos, request, outliers, workers=16):
    """Same values as inputs.kv_vectors, generated in page-aligned blocks on several threads."""
    k = np.empty((n, 4, 256), np.float32)
    v = np.empty((n, 4, 256), np.float32)
    if n == 0:
        return k, v
    blk = 64 * 256
    starts = list(range(first_pos - first_pos % 256, first_pos + n, blk))

    def job(s):
        lo, hi = max(s, first_pos), min(s + blk, first_pos + n)
        kk, vv = I.kv_vectors(config, layer, hi - lo, first_pos=lo, request=request, outlier_frac=outliers)
        k[lo - first_pos:hi - first_pos] = kk
        v[lo - first_pos:hi - first_pos] = vv

    with cf.ThreadPoolExecutor(workers) as ex:
        list(ex.map(job, starts))
    return k, v


class Arena:
    """One contiguous device buffer carved into aligned tensors, with a pinned host mirror."""

    def __init__(self, torch, device):
        self.torch, self.device, self.parts, self.nbytes = torch, device, [], 0

    def add(self, host_array, dtype, shape):
        off = self.nbytes
        nb = int(np.asarray(host_array).nbytes)
        self.parts.append((off, nb, host_array, dtype, shape))
        self.nbytes = (off + nb + 255) // 256 * 256
        return len(self.parts) - 1

    def finalize(self):
        torch = self.torch
        self.dev = torch.empty(max(self.nbytes, 256), dtype=torch.uint8, device=self.device)
        self.host = torch.empty(max(self.nbytes, 256), dtype=torch.uint8).pin_memory()
        hv = self.host.numpy()
        self.views = []
        for off, nb, arr, dtype, shape in self.parts:
            if arr is not None:
                hv[off:off + nb] = np.frombuffer(np.ascontiguousarray(arr).tobytes(), np.uint8)
            self.views.append(self.dev[off:off + nb].view(dtype).view(shape))
        self.dev.copy_(self.host)
        return self.views


class DecodeSetup:
    def __init__(self, w, torch, tq4, device):
        self.w, self.torch, self.tq4 = w, torch, tq4
        self.signs = I.signs(w.config)
        self.ctx = tq4.Context(self.signs)
        self.tables_np = I.request_tables(w)
        self.tables = torch.from_numpy(self.tables_np).to(device)
        self.seq_np = np.array(w.seq_lens, np.int32)
        self.seq = torch.from_numpy(self.seq_np).to(device)
        self.total = int(self.seq_np.sum())
        self.n_q = w.n_q
        self.pools = []
        self.ws = self.ctx.decode_workspace(w.n_req, w.n_q, self.total, device)
        ain, aout = Arena(torch, device), Arena(torch, device)
        qi, ki, vi, oi = [], [], [], []
        for layer in range(w.layers):
            pool = tq4.Context.new_pool(w.pool_pages, device)
            knew_l, vnew_l = [], []
            for r in range(w.n_req):
                first = w.shared_prefix_pages * 256 if r > 0 else 0
                s = int(self.seq_np[r])
                k, v = gen_kv_parallel(w.config, layer, s - first, first, r, w.outlier_frac)
                tt = self.tables[r]
                hist = s - w.n_q - first  # history already in the cache; the last n_q are the step's appends
                for a in range(0, hist, 32768):
                    e = min(a + 32768, hist)
                    self.ctx.encode_append(pool, tt, first + a, torch.from_numpy(k[a:e]).to(device),
                                           torch.from_numpy(v[a:e]).to(device))
                knew_l.append(np.ascontiguousarray(k[hist:]))
                vnew_l.append(np.ascontiguousarray(v[hist:]))
                del k, v
            # the step's new K/V of all requests: [n_req, n_q, 4, 256] fp32
            ki.append(ain.add(np.stack(knew_l), torch.float32, (w.n_req, w.n_q, 4, 256)))
            vi.append(ain.add(np.stack(vnew_l), torch.float32, (w.n_req, w.n_q, 4, 256)))
            qb = I.queries(w.config, layer, (w.n_req, w.n_q, 24, 256))
            qi.append(ain.add(qb, torch.bfloat16, (w.n_req, w.n_q, 24, 256)))
            oi.append(aout.add(np.zeros((w.n_req, w.n_q, 24, 256), np.uint16), torch.bfloat16,
                               (w.n_req, w.n_q, 24, 256)))
            self.pools.append(pool)
        vin, vout = ain.finalize(), aout.finalize()
        self.arena_in, self.arena_out = ain, aout
        self.qs = [vin[i] for i in qi]
        self.knew = [vin[i] for i in ki]
        self.vnew = [vin[i] for i in vi]
        self.outs = [vout[i] for i in oi]
        torch.cuda.synchronize()
        st = self.ctx.status()
        if st != tq4.TQ4_OK:
            raise RuntimeError(f"cache build failed with device status {st}")

    # raw ABI calls (no Python-side allocation) so that the step can be captured
    def attend(self, layer):
        """The step's append and decode of one layer, one call (the timed attention call)."""
        tq4, w = self.tq4, self.w
        rc = tq4.tq4_decode_append_attention(self.ctx.handle, self.pools[layer], w.pool_pages, self.knew[layer],
                                             self.vnew[layer], tq4.DTYPE_F32, self.qs[layer], self.tables,
                                             self.tables.shape[1], self.seq, w.n_req, w.n_q, self.total, SCALE,
                                             self.outs[layer], tq4.DTYPE_BF16, self.ws, self.ws.numel())
        assert rc == 0, rc

    def step(self):
        for layer in range(self.w.layers):
            self.attend(layer)

    def units_per_step(self):
        return self.total * self.w.layers  # attended KV positions x layers

    def kernels_per_step(self):
        # decode + combine per layer; with n_q > 1 a tail-encode kernel as well
        return self.w.layers * (2 if self.w.n_q == 1 else 3)

    def dominant_bytes(self):
        """Algorithmic bytes of one decode launch: the packed history it must read."""
        return self.total * I.H_KV * 2 * 130

    def h2d_d2h(self):
        return self.arena_in.nbytes, self.arena_out.nbytes


class PrefillSetup:
    def __init__(self, w, torch, tq4, device):
        self.w, self.torch, self.tq4 = w, torch, tq4
        self.signs = I.signs(w.config)
        self.ctx = tq4.Context(self.signs)
        self.tables_np = I.request_tables(w)
        self.table = torch.from_numpy(self.tables_np[0]).to(device)
        self.P, self.n = w.prefix_len, w.n_q
        self.pools = []
        self.ws = torch.empty(tq4.tq4_prefill_workspace_bytes(self.n), dtype=torch.uint8, device=device)
        ain, aout = Arena(torch, device), Arena(torch, device)
        idx = []
        for layer in range(w.layers):
            pool = tq4.Context.new_pool(w.pool_pages, device)
            k, v = gen_kv_parallel(w.config, layer, self.P, 0, 0, w.outlier_frac)
            for a in range(0, self.P, 32768):
                e = min(a + 32768, self.P)
                self.ctx.encode_append(pool, self.table, a, torch.from_numpy(k[a:e]).to(device),
                                       torch.from_numpy(v[a:e]).to(device))
            del k, v
            qb = I.queries(w.config, layer, (self.n, 24, 256))
            kb, vb = I.chunk_kv(w.config, layer, self.n)
            idx.append((ain.add(qb, torch.bfloat16, (self.n, 24, 256)),
                        ain.add(kb, torch.bfloat16, (self.n, 4, 256)),
                        ain.add(vb, torch.bfloat16, (self.n, 4, 256)),
                        aout.add(np.zeros((self.n, 24, 256), np.uint16), torch.bfloat16, (self.n, 24, 256))))
            self.pools.append(pool)
        vin, vout = ain.finalize(), aout.finalize()
        self.arena_in, self.arena_out = ain, aout
        self.q = [vin[a] for a, _, _, _ in idx]
        self.kc = [vin[b] for _, b, _, _ in idx]
        self.vc = [vin[c] for _, _, c, _ in idx]
        self.outs = [vout[d] for _, _, _, d in idx]
        torch.cuda.synchronize()
        if self.ctx.status() != tq4.TQ4_OK:
            raise RuntimeError("cache build failed")

    def attend(self, layer):
        tq4, w = self.tq4, self.w
        rc = tq4.tq4_prefill_attention(self.ctx.handle, self.pools[layer], w.pool_pages, self.table,
                                       self.table.numel(), self.P, self.q[layer], self.kc[layer], self.vc[layer],
                                       self.n, SCALE, self.outs[layer], self.ws, self.ws.numel())
        assert rc == 0, rc

    def append(self, layer):
        tq4, w = self.tq4, self.w
        rc = tq4.tq4_encode_append(self.ctx.handle, self.pools[layer], w.pool_pages, self.table,
                                   self.table.numel(), self.P, self.n, self.kc[layer], self.vc[layer],
                                   tq4.DTYPE_BF16)
        assert rc == 0, rc

    def step(self):
        for layer in range(self.w.layers):
            self.attend(layer)
            self.append(layer)

    def units_per_step(self):
        # attended KV positions summed over the chunk's query tokens, x layers
        return self.w.layers * (self.n * self.P + self.n * (self.n + 1) // 2)

    def kernels_per_step(self):
        return self.w.layers * 3

    def dominant_flops(self):
        """Algorithmic FLOPs of one prefill launch (QK^T and PV, causal part only)."""
        att = self.n * self.P + self.n * (self.n + 1) // 2
        return 2 * 2 * 24 * 256 * att

    def h2d_d2h(self):
        return self.arena_in.nbytes, self.arena_out.nbytes


# ---------------------------------------------------------------------------- CPU oracle legs
class OracleSample:
    """The oracle on one layer of the workload (a bounded sample); state is built once."""

    def __init__(self, w):
        from oracle import tq4_oracle as O
        self.O, self.w = O, w
        self.signs = I.signs(w.config)
        self.c, _ = O.codebook()
        self.tables = I.request_tables(w)
        if w.kind == "decode":
            T = min(int(w.seq_lens[0]), 8192)
            self.T = T
            self.k, self.v = gen_kv_parallel(w.config, 0, T, 0, 0, w.outlier_frac)
            self.pool = O.new_pool(w.pool_pages)
            O.encode_append(self.pool, self.tables[0], 0, self.k[:T - w.n_q], self.v[:T - w.n_q],
                            self.signs, self.c)
            self.qf = I.bf16_bits_to_f32(I.queries(w.config, 0, (1, w.n_q, 24, 256)))
            self.sample = (f"1 layer, 1 request, the first {T} positions of the workload's history, "
                           f"n_q={w.n_q}: append of the step's new position(s) + decode attention")
        else:
            P = min(w.prefix_len, 4096)
            self.P = P
            k, v = gen_kv_parallel(w.config, 0, P, 0, 0, 0.0)
            self.pool = O.new_pool(w.pool_pages)
            O.encode_append(self.pool, self.tables[0], 0, k, v, self.signs, self.c)
            qb = I.queries(w.config, 0, (w.n_q, 24, 256))
            kb, vb = I.chunk_kv(w.config, 0, w.n_q)
            self.qf, self.kf, self.vf = (I.bf16_bits_to_f32(a) for a in (qb, kb, vb))
            self.rows = np.arange(0, w.n_q, 256)
            self.sample = f"1 layer, {P}-position prefix, {len(self.rows)} of {w.n_q} query tokens"

    def one(self):
        O, w = self.O, self.w
        if w.kind == "decode":
            T = self.T
            O.encode_append(self.pool, self.tables[0], T - w.n_q, self.k[T - w.n_q:], self.v[T - w.n_q:],
                            self.signs, self.c)
            O.decode_attention(self.pool, self.tables[:1], [T], self.qf, SCALE, self.signs, self.c)
            return T
        O.prefill_attention(self.pool, self.tables[0], self.P, self.qf, self.kf, self.vf, SCALE, self.signs,
                            self.c, rows=self.rows)
        return int(sum(self.P + i + 1 for i in self.rows))

    @staticmethod
    def threads():
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([d.get("num_threads", 1) for d in info] or [1])

    def timed(self, seconds=10.0):
        self.one()
        units, t0 = 0, time.perf_counter()
        while True:
            units += self.one()
            el = time.perf_counter() - t0
            if el >= seconds:
                return units / el, el


def run_reference(args, rank):
    """The reference arm: the CPU oracle itself, on bounded samples of the workload."""
    if rank != 0:
        return
    w = I.WORKLOADS[args.workload]
    orc = OracleSample(w)
    for _ in range(args.warmup):
        orc.one()
    units, t0 = 0, time.perf_counter()
    for _ in range(args.steps):
        units += orc.one()
    el = time.perf_counter() - t0
    value = units / el
    threads = orc.threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / max(args.steps, 1) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Gaussian K/V and queries)",
            "config": dict(workload_config(args.workload, args.gpus), sample=orc.sample),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": orc.sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- main
def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    from compressed_paged_kv_tq4_b200 import tq4

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    w = I.WORKLOADS[args.workload]
    if args.layers:
        import dataclasses
        w = dataclasses.replace(w, layers=args.layers)
    if args.profile:
        args.eager = True
    S = DecodeSetup(w, torch, tq4, device) if w.kind == "decode" else PrefillSetup(w, torch, tq4, device)
    stream = torch.cuda.Stream(device)

    # capture one step through the public ABI
    graph = None
    with torch.cuda.stream(stream):
        S.step()  # eager once (also the first warm-up)
        torch.cuda.synchronize()
        if not args.eager:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                S.step()
    torch.cuda.synchronize()
    run = graph.replay if graph is not None else S.step

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            run()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(args.steps):
                run()
            ev1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, device)
    if S.ctx.status() != tq4.TQ4_OK:
        raise RuntimeError("device status error during timing")
    value = job_value(S.units_per_step(), world, ms)
    if args.profile:
        if rank == 0:
            print(json.dumps({"profile": True, "workload": args.workload, "layers": w.layers, "ms_per_step": ms}))
        return

    # dominant kernel: the attention call, timed alone (graph of the attention launches of all layers)
    hbm, bf16, bf16_sus, peak_kind = peaks()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        torch.cuda.synchronize()
        with torch.cuda.graph(g2, stream=stream):
            for layer in range(w.layers):
                S.attend(layer)
        for _ in range(5):
            g2.replay()
        reps = max(20, min(200, args.steps))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g2.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    att_ms = e0.elapsed_time(e1) / (reps * w.layers)
    if w.kind == "decode":
        ach = S.dominant_bytes() / (att_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": (measured_traffic("decode_q1", S.total) if w.n_q == 1 else
                            measured_traffic("decode_splitk", S.total) if w.name == "verify_2req_229k" else None),
                "kernel": "tq4_decode_append_attention (split-K decode with the append inside it for one "
                          "query token + combine)",
                "launch_ms": att_ms, "peak_source": f"{peak_kind} hbm_gbs"}
    else:
        ach = S.dominant_flops() / (att_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": bf16, "unit": "TFLOP/s", "frac": ach / bf16,
                "traffic": measured_traffic("prefill_tc", 1) if w.name == "prefill_2k_on_32k" else None,
                "kernel": "tq4_prefill_attention (rotate prologue + attention kernel)",
                "launch_ms": att_ms, "peak_source": f"{peak_kind} bf16_tflops (f16 operands: same nominal rate)"}

    # end to end: pinned host inputs in, results out, every step
    h2d, d2h = S.h2d_d2h()
    e2e = None
    if graph is not None:
        ain, aout = S.arena_in, S.arena_out
        n_e2e = max(10, min(args.steps, 200))
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(n_e2e):
                ain.dev.copy_(ain.host, non_blocking=True)     # this step's queries and new K/V
                graph.replay()
                aout.host.copy_(aout.dev, non_blocking=True)   # every layer's attention output
            e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        e2e_ms = max_over_ranks(e2e_ms, dist, device)
        e2e = {"value": job_value(S.units_per_step(), world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms,
               "path": "pinned H2D of the step's queries and new K/V, replay of the captured public C-ABI "
                       "calls, D2H of every layer's output"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        orc = OracleSample(w)
        v, el = orc.timed(10.0)
        cpu = {"value": v, "unit": UNIT, "cores": orc.threads(), "kind": "oracle", "sample": orc.sample,
               "seconds": el}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u4 codes, f16 tensor-core operands, f32 accumulate",
            "data": "synthetic (seeded Gaussian K/V and queries)",
            "config": workload_config(args.workload, world),
            "graph": graph is not None,
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": S.kernels_per_step() * args.steps,
            "clocks": clk.summary(),
            "tokens_per_s": (w.n_req * w.n_q if w.kind == "decode" else w.n_q) * world / (ms * 1e-3),
        }
        print(json.dumps(line), flush=True)
    del graph, g2
    if dist:
        dist.barrier()
        dist.destroy_process_group()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
