#!/usr/bin/env python
"""Benchmark of the TQ4 paged-KV attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--extra LIST]
                    [--impl ours|reference]

One step = one pass of the whole hot path over one batch: for every layer,
tq4_decode_append_attention (the step's new K/V positions appended, then decode
attention over the whole history; with one query token the append runs inside
the decode kernel) for decode workloads, or tq4_prefill_attention followed by
tq4_encode_append of the chunk (prefill workload). The step's launches are
captured once in a CUDA graph through the public C ABI and replayed; the timed
region is exactly K replays between CUDA events, after W warm-up replays.

The headline line is the `--workload` (decode_32k by default, 16 layers of
32,768 positions). The other workloads (`--extra`: the three others and the INT8 arm by default) are
measured in the same run the same way, with as many timed steps as fit in about
two seconds (at most K), and reported under "workloads" in the same JSON line.

Prints one JSON line. Multi-GPU runs (torchrun) are independent replicas: the
path has no exchange step, every rank runs the same workload on its own GPU
and the value is the units of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
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
EXTRA_DEFAULT = ("decode_213k_outliers,verify_2req_229k,shared_prefix_8req_33k,prefill_2k_on_32k,int8_decode_32k,"
                 "tqb3_decode_32k,tqb2_decode_32k")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode_32k", choices=sorted(I.WORKLOADS))
    ap.add_argument("--extra", default=EXTRA_DEFAULT,
                    help="comma-separated workloads measured after the headline one ('none' for none)")
    ap.add_argument("--extra-seconds", type=float, default=2.0, help="timed seconds per extra workload (about)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch without a CUDA graph (profiling)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling only)")
    ap.add_argument("--decode-path", default="default", choices=["default", "warp", "tensor"],
                    help="kernel for 2-4 query tokens (tq4_ctx_set_decode_path); default: the library's")
    ap.add_argument("--profile", action="store_true",
                    help="eager steps of the one workload only: no roofline replay, e2e or CPU leg (ncu captures)")
    return ap.parse_args(argv)


def peaks():
    """(hbm GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained") or d["bf16_tflops"]), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


WORKLOAD_DESC = {
    "decode_32k": "16 layers x 32,768 TQ4 positions, 1 request, 1 bf16 query token, 24 Q / 4 KV heads x 256",
    "decode_213k_outliers": "16 layers x 212,992 TQ4 positions (5% x8 outliers), 1 request, 1 query token",
    "verify_2req_229k": "2 requests (163,840 + 65,536 positions, 64 shared pages), 4 causal query tokens each, "
                        "16 layers (timed ungrouped; the grouped decode is timed beside it)",
    "shared_prefix_8req_33k": "8 requests of 33,792 positions sharing their first 32,768 (128 pages), 1 query token "
                              "each, 16 layers, grouped decode (the shared pages read once; the ungrouped decode "
                              "is timed beside it)",
    "prefill_2k_on_32k": "2,048 causal bf16 query tokens on a 32,768-position TQ4 prefix + the chunk, 16 layers "
                         "(packed prefix; direct inverse reconstruction timed beside it)",
    "single_layer_2k": "1 layer, 2,048 TQ4 positions, 1 query token",
    "int8_decode_32k": "uniform INT8 comparison arm: 16 layers x 32,768 INT8 positions (2,064 B per "
                       "layer-position), 1 request, 1 bf16 query token, append of 1 position per layer",
    "tqb3_decode_32k": "3-bit variant: 16 layers x 32,768 positions (784 B per layer-position), 1 request, "
                       "1 bf16 query token, append of 1 position per layer",
    "tqb2_decode_32k": "2-bit variant: 16 layers x 32,768 positions (528 B per layer-position), 1 request, "
                       "1 bf16 query token, append of 1 position per layer",
}


def workload_config(name, world):
    """The `config` object of the JSON line (the same for both arms)."""
    w = I.WORKLOADS[name]
    per_pos = {"decode_int8": 2064, "decode_tqb2": 528, "decode_tqb3": 784}.get(w.kind, 1040)
    return {"workload": f"{name}: {WORKLOAD_DESC[name]}", "append_per_layer": w.append_per_step,
            "pool_pages": w.pool_pages, "page_positions": 256,
            "l2": "inputs larger than L2: packed KV read per step is "
                  f"{w.layers * sum(w.seq_lens) * per_pos / 1e6:.0f} MB vs 126 MB L2",
            "parallelism": f"replicas x{world}"}


# ---------------------------------------------------------------------------- measured DRAM traffic
# DRAM bytes (read + write) per launch of each workload's dominant kernel, from one
# ncu capture of that workload (summarised under profiles/). The figures count only
# while the kernel sources hash to the value they had when the counters were taken.
MEASURED_TRAFFIC_SOURCES = "7628c67e128fb178515366d470678ff947cab69f7aea0ee838a90e1407f5a6d7"
MEASURED_TRAFFIC = {
    "decode_32k": 34_219_008,              # decode_q1_kernel<0,4>: 34,183,936 read + 35,072 written
    "decode_213k_outliers": 225_226_496,   # decode_q1_kernel<0,4>: 221,925,888 read + 3,300,608 written
    "verify_2req_229k": 224_868_096,       # decode_splitk_kernel<3,3>: 221,704,960 read + 3,163,136 written
    "shared_prefix_8req_33k": 43_067_392,  # decode_splitk_kernel<1,6> (grouped): 42,843,136 read + 224,256 written
    "int8_decode_32k": 68_552_448,         # decode_splitk_kernel<1,1,INT8>: 67,694,080 read + 858,368 written
    "prefill_2k_on_32k": 203_590_912,      # prefill_tc_kernel: 102,009,600 read + 101,581,312 written (segment partials)
    "tqb3_decode_32k": 25_804_288,         # decode_q1_kernel<0,3>: 25,802,240 read + 2,048 written
    "tqb2_decode_32k": 17_408_512,         # decode_q1_kernel<0,2>: 17,408,512 read + 0 written
}


def sources_digest():
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "compressed_paged_kv_tq4_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cuh")) + glob.glob(os.path.join(csrc, "*.cu"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload):
    """DRAM bytes per launch of the workload's dominant kernel, or None if the kernel
    sources changed since the capture."""
    if workload not in MEASURED_TRAFFIC:
        return None
    try:
        if sources_digest() != MEASURED_TRAFFIC_SOURCES:
            return None
    except OSError:
        return None
    return MEASURED_TRAFFIC[workload]


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


# ---------------------------------------------------------------------------- device data
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
    """One decode workload on the device: every layer's pool (history encoded by
    tq4_encode_append from K/V drawn on the device with the workload's law), page
    tables, lengths, and the step's inputs (queries, new K/V) and outputs in one
    arena with a pinned host mirror."""

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
        # requests sharing their first pages: the grouped decode (shared pages read once)
        # times the workload when w.grouped, else it is timed beside the plain decode
        self.has_groups = w.shared_prefix_pages > 0 and w.n_req > 1
        self.has_alt = self.has_groups
        self.shared = self.has_groups and w.grouped
        self.leader = np.zeros(w.n_req, np.int32)
        self.pages = np.full(w.n_req, w.shared_prefix_pages, np.int32)
        self.ws = self.ctx.decode_workspace(w.n_req, w.n_q, self.total, device)
        if self.has_groups:
            nbytes = tq4.tq4_decode_shared_workspace_bytes(self.ctx.handle, w.n_req, w.n_q, self.total,
                                                           self.tables.shape[1], self.leader, self.pages)
            self.ws_shared = torch.empty(nbytes, dtype=torch.uint8, device=device)
        ain, aout = Arena(torch, device), Arena(torch, device)
        qi, ki, vi, oi = [], [], [], []
        for layer in range(w.layers):
            pool = tq4.Context.new_pool(w.pool_pages, device)
            knew_l, vnew_l = [], []
            for r in range(w.n_req):
                first = w.shared_prefix_pages * 256 if r > 0 else 0
                s = int(self.seq_np[r])
                k, v = I.kv_vectors_device(w.config, layer, s - first, request=r, outlier_frac=w.outlier_frac,
                                           device=device)
                hist = s - w.n_q - first  # history already in the cache; the last n_q are the step's appends
                self.ctx.encode_append(pool, self.tables[r], first, k[:hist], v[:hist])
                knew_l.append(k[hist:].cpu().numpy())
                vnew_l.append(v[hist:].cpu().numpy())
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
        if self.shared:
            rc = tq4.tq4_decode_attention_shared(self.ctx.handle, self.pools[layer], w.pool_pages, self.knew[layer],
                                                 self.vnew[layer], tq4.DTYPE_F32, self.qs[layer], self.tables,
                                                 self.tables.shape[1], self.seq, w.n_req, w.n_q, self.total,
                                                 self.leader, self.pages, SCALE, self.outs[layer], tq4.DTYPE_BF16,
                                                 self.ws_shared, self.ws_shared.numel())
        else:
            rc = tq4.tq4_decode_append_attention(self.ctx.handle, self.pools[layer], w.pool_pages, self.knew[layer],
                                                 self.vnew[layer], tq4.DTYPE_F32, self.qs[layer], self.tables,
                                                 self.tables.shape[1], self.seq, w.n_req, w.n_q, self.total, SCALE,
                                                 self.outs[layer], tq4.DTYPE_BF16, self.ws, self.ws.numel())
        assert rc == 0, rc

    def step(self):
        for layer in range(self.w.layers):
            self.attend(layer)

    def flip(self):   # grouped <-> ungrouped decode
        self.shared = not self.shared

    def alt_name(self):   # the path not timed as the workload's
        return "ungrouped (tq4_decode_append_attention)" if self.shared else "grouped (tq4_decode_attention_shared)"

    def alternatives(self):
        """The workload's other paths on the same inputs: (name, enter, leave)."""
        alts = []
        if self.n_q > 1 and not self.shared:   # 2-4 tokens: the tensor-memory kernel beside the default one
            tq4 = self.tq4
            alts.append(("tcgen05 tensor-memory split-K kernel (decode path TQ4_DECODE_PATH_TENSOR_MEMORY)",
                         lambda: self.ctx.set_decode_path(tq4.DECODE_PATH_TENSOR_MEMORY),
                         lambda: self.ctx.set_decode_path(tq4.DECODE_PATH_WARP_MMA)))
        if self.has_groups:
            alts.append((self.alt_name(), self.flip, self.flip))
        return alts

    def units_per_step(self):
        return self.total * self.w.layers  # attended KV positions x layers

    def kernels_per_step(self):
        # decode + combine per layer; with n_q > 1 a tail-encode kernel as well
        return self.w.layers * (2 if self.w.n_q == 1 else 3)

    def roofline(self, att_ms, peaks_):
        """Dominant call: one layer's tq4_decode_append_attention (tq4_decode_attention_shared
        when requests share pages); algorithmic bytes = the packed history it must read,
        1,040 B per distinct layer-position (shared pages count once)."""
        hbm = peaks_[0]
        distinct = self.total - (self.w.n_req - 1) * self.w.shared_prefix_pages * I.PAGE if self.shared else self.total
        nbytes = distinct * I.H_KV * 2 * 130
        ach = nbytes / (att_ms * 1e-3) / 1e9
        kernel = ("tq4_decode_attention_shared with its append (tail encode + one split-K launch of group and "
                  "private items + combine)" if self.shared else
                  "tq4_decode_append_attention (split-K decode with the append inside it for one query token "
                  "+ combine)")
        return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": measured_traffic(self.w.name),
                "kernel": kernel,
                "algorithmic_bytes_per_launch": nbytes, "launch_ms": att_ms,
                "peak_source": f"{peaks_[3]} hbm_gbs"}

    def h2d_d2h(self):
        return self.arena_in.nbytes, self.arena_out.nbytes

    def tokens_per_step(self):
        return self.w.n_req * self.w.n_q


class Int8DecodeSetup(DecodeSetup):
    """The uniform INT8 comparison arm on a decode workload: each layer's pool holds
    the INT8-encoded history; a step appends the new position with
    tq4_int8_encode_append and runs tq4_int8_decode_attention, per layer."""

    def __init__(self, w, torch, tq4, device):
        self.w, self.torch, self.tq4 = w, torch, tq4
        self.ctx = tq4.Context(I.signs(w.config))
        self.tables_np = I.request_tables(w)
        self.tables = torch.from_numpy(self.tables_np).to(device)
        self.seq_np = np.array(w.seq_lens, np.int32)
        self.seq = torch.from_numpy(self.seq_np).to(device)
        self.total = int(self.seq_np.sum())
        self.start = int(self.seq_np[0]) - w.n_q
        if w.n_req != 1:
            raise ValueError("the INT8 arm's bench workload has one request")
        self.pools = []
        self.ws = self.ctx.decode_workspace(w.n_req, w.n_q, self.total, device)
        ain, aout = Arena(torch, device), Arena(torch, device)
        qi, ki, vi, oi = [], [], [], []
        for layer in range(w.layers):
            pool = tq4.Context.new_int8_pool(w.pool_pages, device)
            k, v = I.kv_vectors_device(w.config, layer, self.total, outlier_frac=w.outlier_frac, device=device)
            self.ctx.int8_encode_append(pool, self.tables[0], 0, k[:self.start], v[:self.start])
            ki.append(ain.add(k[self.start:].cpu().numpy(), torch.float32, (w.n_q, 4, 256)))
            vi.append(ain.add(v[self.start:].cpu().numpy(), torch.float32, (w.n_q, 4, 256)))
            del k, v
            qb = I.queries(w.config, layer, (1, w.n_q, 24, 256))
            qi.append(ain.add(qb, torch.bfloat16, (1, w.n_q, 24, 256)))
            oi.append(aout.add(np.zeros((1, w.n_q, 24, 256), np.uint16), torch.bfloat16, (1, w.n_q, 24, 256)))
            self.pools.append(pool)
        vin, vout = ain.finalize(), aout.finalize()
        self.arena_in, self.arena_out = ain, aout
        self.qs = [vin[i] for i in qi]
        self.knew = [vin[i] for i in ki]
        self.vnew = [vin[i] for i in vi]
        self.outs = [vout[i] for i in oi]
        torch.cuda.synchronize()
        if self.ctx.status() != tq4.TQ4_OK:
            raise RuntimeError("INT8 cache build failed")

    def alternatives(self):   # the INT8 arm has one kernel path
        return []

    def attend(self, layer):
        """The step's append and decode of one layer: two calls on the INT8 arm."""
        tq4, w = self.tq4, self.w
        rc = tq4.tq4_int8_encode_append(self.ctx.handle, self.pools[layer], w.pool_pages, self.tables[0],
                                        self.tables.shape[1], self.start, w.n_q, self.knew[layer], self.vnew[layer],
                                        tq4.DTYPE_F32)
        assert rc == 0, rc
        rc = tq4.tq4_int8_decode_attention(self.ctx.handle, self.pools[layer], w.pool_pages, self.qs[layer],
                                           self.tables, self.tables.shape[1], self.seq, w.n_req, w.n_q, self.total,
                                           SCALE, self.outs[layer], tq4.DTYPE_BF16, self.ws, self.ws.numel())
        assert rc == 0, rc

    def kernels_per_step(self):
        return self.w.layers * 3   # encode, decode, combine

    def roofline(self, att_ms, peaks_):
        """Dominant call: one layer's append + INT8 decode; algorithmic bytes = the INT8
        history it must read (2,064 B per attended layer-position)."""
        hbm = peaks_[0]
        nbytes = self.total * I.H_KV * 2 * 258
        ach = nbytes / (att_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": measured_traffic(self.w.name),
                "kernel": "tq4_int8_encode_append + tq4_int8_decode_attention (split-K + combine)",
                "algorithmic_bytes_per_launch": nbytes, "launch_ms": att_ms, "peak_source": f"{peaks_[3]} hbm_gbs"}


class TqbDecodeSetup(Int8DecodeSetup):
    """The 2- or 3-bit variant on a decode workload: each layer's pool holds the
    history in the narrower format; a step is tq4_tqb_decode_append_attention per
    layer (the new position appended inside the one-token decode kernel)."""

    def __init__(self, w, torch, tq4, device):
        self.w, self.torch, self.tq4 = w, torch, tq4
        self.bits = 2 if w.kind == "decode_tqb2" else 3
        self.ctx = tq4.Context(I.signs(w.config))
        self.tables_np = I.request_tables(w)
        self.tables = torch.from_numpy(self.tables_np).to(device)
        self.seq_np = np.array(w.seq_lens, np.int32)
        self.seq = torch.from_numpy(self.seq_np).to(device)
        self.total = int(self.seq_np.sum())
        self.start = int(self.seq_np[0]) - w.n_q
        if w.n_req != 1:
            raise ValueError("the variants' bench workloads have one request")
        self.pools = []
        self.ws = self.ctx.decode_workspace(w.n_req, w.n_q, self.total, device)
        ain, aout = Arena(torch, device), Arena(torch, device)
        qi, ki, vi, oi = [], [], [], []
        for layer in range(w.layers):
            pool = tq4.Context.new_tqb_pool(self.bits, w.pool_pages, device)
            k, v = I.kv_vectors_device(w.config, layer, self.total, outlier_frac=w.outlier_frac, device=device)
            self.ctx.tqb_encode_append(self.bits, pool, self.tables[0], 0, k[:self.start], v[:self.start])
            ki.append(ain.add(k[self.start:].cpu().numpy(), torch.float32, (w.n_q, 4, 256)))
            vi.append(ain.add(v[self.start:].cpu().numpy(), torch.float32, (w.n_q, 4, 256)))
            del k, v
            qb = I.queries(w.config, layer, (1, w.n_q, 24, 256))
            qi.append(ain.add(qb, torch.bfloat16, (1, w.n_q, 24, 256)))
            oi.append(aout.add(np.zeros((1, w.n_q, 24, 256), np.uint16), torch.bfloat16, (1, w.n_q, 24, 256)))
            self.pools.append(pool)
        vin, vout = ain.finalize(), aout.finalize()
        self.arena_in, self.arena_out = ain, aout
        self.qs = [vin[i] for i in qi]
        self.knew = [vin[i] for i in ki]
        self.vnew = [vin[i] for i in vi]
        self.outs = [vout[i] for i in oi]
        torch.cuda.synchronize()
        if self.ctx.status() != tq4.TQ4_OK:
            raise RuntimeError(f"{self.bits}-bit cache build failed")

    def kernels_per_step(self):
        # decode (append fused) + combine per layer; with n_q > 1 a tail-encode kernel as well
        return self.w.layers * (2 if self.w.n_q == 1 else 3)

    def attend(self, layer):
        """The step's append and decode of one layer: one fused call on the variant."""
        tq4, w = self.tq4, self.w
        rc = tq4.tq4_tqb_decode_append_attention(self.ctx.handle, self.bits, self.pools[layer], w.pool_pages,
                                                 self.knew[layer], self.vnew[layer], tq4.DTYPE_F32, self.qs[layer],
                                                 self.tables, self.tables.shape[1], self.seq, w.n_req, w.n_q,
                                                 self.total, SCALE, self.outs[layer], tq4.DTYPE_BF16, self.ws,
                                                 self.ws.numel())
        assert rc == 0, rc

    def roofline(self, att_ms, peaks_):
        """Dominant call: one layer's append + decode of the variant; algorithmic bytes =
        the packed history it must read (528 B or 784 B per attended layer-position)."""
        hbm = peaks_[0]
        nbytes = self.total * I.H_KV * 2 * (32 * self.bits + 2)
        ach = nbytes / (att_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": measured_traffic(self.w.name),
                "kernel": f"tq4_tqb_decode_append_attention, {self.bits} bits (decode_q1_kernel<0,{self.bits}> with the "
                          "append fused + combine)",
                "algorithmic_bytes_per_launch": nbytes, "launch_ms": att_ms, "peak_source": f"{peaks_[3]} hbm_gbs"}


class PrefillSetup:
    """The prefill workload on the device: every layer's pool holds the TQ4 prefix
    (encoded from K/V drawn on the device); the chunk's queries and K/V are seeded
    bf16 inputs in an arena with a pinned host mirror."""

    def __init__(self, w, torch, tq4, device):
        self.w, self.torch, self.tq4 = w, torch, tq4
        self.signs = I.signs(w.config)
        self.ctx = tq4.Context(self.signs)
        self.tables_np = I.request_tables(w)
        self.table = torch.from_numpy(self.tables_np[0]).to(device)
        self.P, self.n = w.prefix_len, w.n_q
        self.pools = []
        # room for the direct-reconstruction variant too (timed beside the packed path)
        self.reconstruct = False
        self.has_alt = True
        self.ws = torch.empty(tq4.tq4_prefill_reconstructed_workspace_bytes(self.P, self.n), dtype=torch.uint8,
                              device=device)
        ain, aout = Arena(torch, device), Arena(torch, device)
        idx = []
        for layer in range(w.layers):
            pool = tq4.Context.new_pool(w.pool_pages, device)
            k, v = I.kv_vectors_device(w.config, layer, self.P, outlier_frac=w.outlier_frac, device=device)
            self.ctx.encode_append(pool, self.table, 0, k, v)
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
        fn = tq4.tq4_prefill_attention_reconstructed if self.reconstruct else tq4.tq4_prefill_attention
        rc = fn(self.ctx.handle, self.pools[layer], w.pool_pages, self.table, self.table.numel(), self.P,
                self.q[layer], self.kc[layer], self.vc[layer], self.n, SCALE, self.outs[layer], tq4.DTYPE_BF16,
                self.ws, self.ws.numel())
        assert rc == 0, rc

    def flip(self):   # packed prefix <-> direct inverse reconstruction
        self.reconstruct = not self.reconstruct

    def alt_name(self):
        return ("packed prefix (tq4_prefill_attention)" if self.reconstruct else
                "direct inverse reconstruction (tq4_prefill_attention_reconstructed: dense prefix rows, then "
                "the same attention kernel)")

    def alternatives(self):
        return [(self.alt_name(), self.flip, self.flip)]

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

    def roofline(self, att_ms, peaks_):
        """Dominant call: one layer's tq4_prefill_attention; algorithmic FLOPs =
        2 * 2 * 256 per visible (query row, position) pair (QK^T and PV, causal part
        only). The attention launches are timed back to back for tens of ms, so the
        sustained bf16 figure is the peak."""
        att = self.n * self.P + self.n * (self.n + 1) // 2
        flops = 2 * 2 * 24 * 256 * att
        ach = flops / (att_ms * 1e-3) / 1e12
        sus, burst = peaks_[2], peaks_[1]
        return {"bound": "tensor", "achieved": ach, "peak": sus, "unit": "TFLOP/s", "frac": ach / sus,
                "frac_of_burst_peak": ach / burst, "peak_burst": burst,
                "traffic": measured_traffic(self.w.name),
                "kernel": "tq4_prefill_attention (rotate prologue + tcgen05 attention kernel)",
                "algorithmic_flops_per_launch": flops, "launch_ms": att_ms,
                "peak_source": f"{peaks_[3]} bf16_tflops_sustained (f16 operands: same nominal rate)"}

    def h2d_d2h(self):
        return self.arena_in.nbytes, self.arena_out.nbytes

    def tokens_per_step(self):
        return self.n


# ---------------------------------------------------------------------------- CPU oracle legs
def _oracle_kv(config, n, outliers):
    """The workload's K/V for positions [0, n) from the numpy generator, a page-aligned
    block at a time on a few threads (same values as inputs.kv_vectors)."""
    import concurrent.futures as cf
    k = np.empty((n, 4, 256), np.float32)
    v = np.empty((n, 4, 256), np.float32)
    blk = 64 * 256

    def job(s):
        e = min(s + blk, n)
        k[s:e], v[s:e] = I.kv_vectors(config, 0, e - s, first_pos=s, outlier_frac=outliers)

    with cf.ThreadPoolExecutor(8) as ex:
        list(ex.map(job, range(0, n, blk)))
    return k, v


class OracleSample:
    """The oracle on one layer of the workload (a bounded sample); state is built once."""

    def __init__(self, w, decode_positions=8192):
        from oracle import tq4_oracle as O
        self.O, self.w = O, w
        self.signs = I.signs(w.config)
        self.c, _ = O.codebook()
        self.tables = I.request_tables(w)
        if w.kind == "decode_int8":
            raise ValueError("the oracle leg times the TQ4 workloads")
        if w.kind == "decode":
            T = min(int(w.seq_lens[0]), decode_positions)
            self.T = T
            self.k, self.v = _oracle_kv(w.config, T, w.outlier_frac)
            self.pool = O.new_pool(w.pool_pages)
            O.encode_append(self.pool, self.tables[0], 0, self.k[:T - w.n_q], self.v[:T - w.n_q],
                            self.signs, self.c)
            self.qf = I.bf16_bits_to_f32(I.queries(w.config, 0, (1, w.n_q, 24, 256)))
            self.sample = (f"1 layer, 1 request, the first {T} positions of the workload's history, "
                           f"n_q={w.n_q}: append of the step's new position(s) + decode attention")
        else:
            P = min(w.prefix_len, 4096)
            self.P = P
            k, v = _oracle_kv(w.config, P, 0.0)
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
    def cores():
        """Threads the oracle ran on: its fp64 matrix products use the BLAS pool; the
        per-head attention loop is Python on one thread."""
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = max([d.get("num_threads", 1) for d in info] or [1])
        return {"cores": blas, "host_cores": os.cpu_count(),
                "threads_note": f"{blas} BLAS threads for the fp64 matrix products (rotation, K q); the per-head "
                                "attention loop runs on one Python thread"}

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
    # a decode step's sample shrinks with the step count so that the run stays within minutes
    T = max(1024, min(8192, (8192 * 400 // max(1, args.steps + args.warmup)) // 256 * 256))
    orc = OracleSample(w, decode_positions=T)
    for _ in range(args.warmup):
        orc.one()
    units, t0 = 0, time.perf_counter()
    for _ in range(args.steps):
        units += orc.one()
    el = time.perf_counter() - t0
    value = units / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / max(args.steps, 1) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Gaussian K/V and queries)",
            "config": dict(workload_config(args.workload, args.gpus), sample=orc.sample),
            "cpu_baseline": dict({"value": value, "unit": UNIT, "kind": "oracle", "sample": orc.sample},
                                 **orc.cores()),
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- GPU measurement
def measure_workload(name, args, torch, tq4, device, dist, world, steps, headline):
    """Build one workload, capture its step as a CUDA graph, time `steps` replays,
    then the dominant attention call alone and the end-to-end path (graphed and eager)."""
    w = I.WORKLOADS[name]
    if args.layers:
        import dataclasses
        w = dataclasses.replace(w, layers=args.layers)
    S = {"decode": DecodeSetup, "decode_int8": Int8DecodeSetup, "decode_tqb2": TqbDecodeSetup,
         "decode_tqb3": TqbDecodeSetup, "prefill": PrefillSetup}[w.kind](w, torch, tq4, device)
    if args.decode_path != "default":
        S.ctx.set_decode_path(tq4.DECODE_PATH_WARP_MMA if args.decode_path == "warp" else tq4.DECODE_PATH_TENSOR_MEMORY)
    stream = torch.cuda.Stream(device)
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
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            run()
        ev0.record(stream)
        run()
        ev1.record(stream)
    torch.cuda.synchronize()
    if not headline:   # as many steps as fit in about --extra-seconds, at most K, at least 3
        est = ev0.elapsed_time(ev1)
        steps = int(max(3, min(steps, args.extra_seconds * 1e3 / max(est, 1e-3))))
    if dist:
        t = torch.tensor([steps], dtype=torch.int64, device=device)   # every rank times the same steps
        dist.all_reduce(t, op=dist.ReduceOp.MIN)
        steps = int(t.item())
        dist.barrier()
    with ClockSampler(device.index) as clk:
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(steps):
                run()
            ev1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, dist, device)
    if S.ctx.status() != tq4.TQ4_OK:
        raise RuntimeError(f"{name}: device status error during timing")
    res = {"value": job_value(S.units_per_step(), world, ms), "unit": UNIT, "ms_per_step": ms, "steps": steps,
           "tokens_per_s": S.tokens_per_step() * world / (ms * 1e-3),
           "gpu_launches": S.kernels_per_step() * steps, "clocks": clk.summary(), "graph": graph is not None}
    if args.profile:
        return res

    # dominant call: the attention call alone (a graph of the attention launches of all layers)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        torch.cuda.synchronize()
        with torch.cuda.graph(g2, stream=stream):
            for layer in range(w.layers):
                S.attend(layer)
        for _ in range(5):
            g2.replay()
        reps = max(10, min(200, steps))
        ev0.record(stream)
        for _ in range(reps):
            g2.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    att_ms = ev0.elapsed_time(ev1) / (reps * w.layers)
    res["roofline"] = S.roofline(att_ms, peaks())
    others = []
    for name, enter, leave in (S.alternatives() if hasattr(S, "alternatives") else []):
        enter()   # the workload's other path on the same inputs, timed the same way
        g3 = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            torch.cuda.synchronize()
            with torch.cuda.graph(g3, stream=stream):
                for layer in range(w.layers):
                    S.attend(layer)
            for _ in range(5):
                g3.replay()
            ev0.record(stream)
            for _ in range(reps):
                g3.replay()
            ev1.record(stream)
        torch.cuda.synchronize()
        del g3
        leave()
        others.append({"path": name, "launch_ms": ev0.elapsed_time(ev1) / (reps * w.layers)})
    if others:
        res["roofline"]["other_path"] = others[0]
        if len(others) > 1:
            res["roofline"]["other_paths"] = others

    # end to end through the public API: pinned host inputs in, every layer's output out, each step
    h2d, d2h = S.h2d_d2h()
    ain, aout = S.arena_in, S.arena_out
    e2e = {"unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
    for label, fn in (("graph", graph.replay if graph is not None else None), ("eager", S.step)):
        if fn is None:
            continue
        n = max(3, min(steps, 200 if label == "graph" else 50))
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(n):
                ain.dev.copy_(ain.host, non_blocking=True)     # this step's queries and new K/V
                fn()
                aout.host.copy_(aout.dev, non_blocking=True)   # every layer's attention output
            ev1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(ev0.elapsed_time(ev1) / n, dist, device)
        if label == "graph":
            e2e.update(value=job_value(S.units_per_step(), world, e_ms), ms_per_step=e_ms,
                       path="pinned H2D of the step's queries and new K/V, replay of the captured public C-ABI "
                            "calls, D2H of every layer's output")
        else:
            e2e["eager"] = {"value": job_value(S.units_per_step(), world, e_ms), "ms_per_step": e_ms,
                            "path": "the same copies around the calls made one by one through the ctypes binding "
                                    "(argument checks, planning and tensor-map encoding on every call)"}
    if "value" not in e2e:   # eager-only runs
        e2e.update(value=e2e["eager"]["value"], ms_per_step=e2e["eager"]["ms_per_step"])
    res["e2e"] = e2e
    if S.ctx.status() != tq4.TQ4_OK:
        raise RuntimeError(f"{name}: device status error")
    del graph, g2, S
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def finish(line, dist):
    """Print the line (rank 0) and leave the process group once."""
    if line is not None:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- main
def main(argv=None, measure=None):
    """`measure(name, args, dist, world, steps, headline) -> dict` replaces the GPU
    measurement when given (the multi-rank path is tested on CPU ranks that way)."""
    args = parse(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one process per GPU "
                         "with torchrun (python -m torch.distributed.run --nproc-per-node N ... --gpus N)")
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    dist = None
    if measure is None:
        from compressed_paged_kv_tq4_b200 import tq4
        torch.cuda.set_device(local)
        device = torch.device("cuda", local)
        backend = "nccl"
    else:
        tq4, device, backend = None, torch.device("cpu"), "gloo"
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))

    def run(name, steps, headline):
        if measure is not None:
            return measure(name, args, dist, world, steps, headline)
        return measure_workload(name, args, torch, tq4, device, dist, world, steps, headline)

    head = run(args.workload, args.steps, True)
    extras = {}
    if not args.profile:
        for name in [x for x in args.extra.split(",") if x and x != "none" and x != args.workload]:
            extras[name] = dict(run(name, args.steps, False), config=workload_config(name, world))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile and measure is None:
        orc = OracleSample(I.WORKLOADS[args.workload])
        v, el = orc.timed(10.0)
        cpu = dict({"value": v, "unit": UNIT, "kind": "oracle", "sample": orc.sample, "seconds": el}, **orc.cores())

    line = None
    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": head["steps"],
                "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "u4 codes, f16 tensor-core operands, f32 accumulate",
                "data": "synthetic (seeded Gaussian K/V and queries)",
                "config": workload_config(args.workload, world),
                "graph": head.get("graph"), "roofline": head.get("roofline"), "cpu_baseline": cpu,
                "e2e": head.get("e2e"), "gpu_launches": head.get("gpu_launches"), "clocks": head.get("clocks"),
                "tokens_per_s": head.get("tokens_per_s"), "workloads": extras}
    finish(line, dist)


if __name__ == "__main__":
    main()
