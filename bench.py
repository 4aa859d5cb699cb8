"""Benchmark of one paged decode step on B200.

A step is the whole hot path over one batch: [copy_blocks of the step's
copy-on-write pairs, if the workload has any] -> reshape_and_cache of one new
token per sequence -> paged_attn_decode over every cached token.  The default
workload is the OPT-13B-shaped decode layer (64 sequences, 40 heads x 128,
fp16, block size 16, context lengths U[1, 2048], 16k-block pool).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is algorithmic bytes per step
(KV of valid tokens + q + out + table entries + lengths, plus the scatter's
and the copies' bytes) divided by the device time per step, summed over
ranks; inputs are resident in HBM and larger than L2.  ``e2e`` is the same
metric with the step's inputs copied from pinned host memory and the output
copied back inside the timed region, pipelined over two buffer sets and a copy
stream per direction (``e2e.serial_value``: one after the other).
``--impl reference`` times the CPU oracle (float64) on the host's cores on a
bounded sample of the same workload.  Under torchrun each rank runs its own
batch (weak scaling, no collective on the data path); the time is the maximum
over ranks.

Other configurations: the other decode workloads by name (``--prefix-aware``
decodes shared prompts with the shared-prefix call); ``--config prefill``
(a chunk's scatter + the tensor-core prefill, in TFLOP/s against the measured
bf16 throughput); ``--config prefill_fp8`` (the same over an E4M3 cache: the
quantising scatter, the widening gather and the prefill); ``--config swap`` (blocks out to pinned host memory and back,
in GB/s against the copy engines' rate measured in the same run).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_324_b200 import workload as wl  # noqa: E402

METRIC = "paged decode attention KV GB/s and % of B200 HBM peak; sequences/sec"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1000 * 1000
FALLBACK_HBM_GBS = 6650.0
# DRAM traffic of one paged_decode_kernel + reduce launch measured by ncu
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by workload, valid only
# for the decode kernel source it was measured on (sha256 prefix of decode.cu).
NCU_TRAFFIC = {
    "opt13b": {"bytes_per_launch": 1_313_689_344, "kernel_sha": "1e2ef54f9309f55c",
               "capture": "ncu, opt13b_compact (the same sequences, pool cut to the blocks in use)"},
    "gqa": {"bytes_per_launch": 1_222_165_760, "kernel_sha": "1e2ef54f9309f55c",
            "capture": "ncu, gqa_compact (the same sequences, pool cut to the blocks in use)"},
    "fp8": {"bytes_per_launch": 1_116_366_848, "kernel_sha": "1e2ef54f9309f55c",
            "capture": "ncu, fp8_compact (the same sequences, 512-token partitions)"},
}


# the same for the prefill calls (every kernel of one call, summed), keyed on the sha256 prefix of
# prefill.cu followed by prefill_fp8.cu, on the prefill workload
PREFILL_TRAFFIC = {
    "prefill": {"bytes_per_launch": 823_833_856, "kernel_sha": "bcbb51e41e176572",
                "capture": "ncu, prefill workload: v_absmax_kernel + v_narrow_kernel + paged_prefill_kernel"},
    "prefill_fp8": {"bytes_per_launch": 820_305_408, "kernel_sha": "bcbb51e41e176572",
                    "capture": "ncu, prefill workload over an E4M3 cache: widen_blocks_kernel + paged_prefill_kernel"},
}


def prefill_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("prefill.cu", "prefill_fp8.cu"):
        h.update(open(os.path.join(ROOT, "paged_kv_cache_324_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def decode_source_sha() -> str:
    p = os.path.join(ROOT, "paged_kv_cache_324_b200", "csrc", "decode.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = float(json.load(open(p))["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; no setting is changed)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def report(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# device-resident workload
# ---------------------------------------------------------------------------

class DeviceStep:
    """A workload's pools and inputs on one GPU, and the calls of one step."""

    def __init__(self, w: wl.DecodeWorkload, dev, partition_size: int = 0, prefix_aware: bool = False):
        import torch
        from paged_kv_cache_324_b200 import binding as B
        self.w, self.dev, self.B, self.torch = w, dev, B, torch
        self.stream = torch.cuda.current_stream(dev)
        t16 = {"f16": torch.float16, "bf16": torch.bfloat16}

        def up(bits, dtype):
            if dtype == "e4m3":
                return torch.from_numpy(np.ascontiguousarray(bits)).to(dev)
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(t16[dtype])

        self.up = up
        self.k_pool = up(w.initial_pool("k"), w.kv_dtype)
        self.v_pool = up(w.initial_pool("v"), w.kv_dtype)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        for op in w.setup:   # build the cache with the library's own kernels
            if isinstance(op, wl.Scatter):
                B.reshape_and_cache(up(op.k, w.src_dtype), up(op.v, w.src_dtype), self.k_pool, self.v_pool,
                                    torch.from_numpy(op.slots).to(dev), float(w.k_scale), float(w.v_scale),
                                    device_error=self.err)
            else:
                B.copy_blocks(self.k_pool, self.v_pool, torch.from_numpy(op.pairs).to(dev), device_error=self.err)
        sc = w.step_scatter
        self.host = {  # the step's inputs, as raw bits
            "q": w.q, "k_new": sc.k, "v_new": sc.v, "slots": sc.slots, "tables": w.block_tables,
            "lens": w.context_lens,
        }
        if w.step_copy is not None:
            self.host["pairs"] = w.step_copy.pairs
        self.d = {
            "q": up(w.q, w.q_dtype), "k_new": up(sc.k, w.src_dtype), "v_new": up(sc.v, w.src_dtype),
            "slots": torch.from_numpy(sc.slots).to(dev), "tables": torch.from_numpy(w.block_tables).to(dev),
            "lens": torch.from_numpy(w.context_lens).to(dev),
        }
        if "pairs" in self.host:
            self.d["pairs"] = torch.from_numpy(self.host["pairs"]).to(dev)
        self.out = torch.empty_like(self.d["q"])
        ws = B.decode_workspace_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.kv_dtype,
                                      w.block_size, w.max_context_len, partition_size)
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        self.partition_arg = partition_size
        self.partition = B.decode_partition_size(w.num_seqs, w.num_kv_heads, w.head_dim, w.kv_dtype, w.block_size,
                                                 w.max_context_len, partition_size)
        self.prefix_aware = prefix_aware
        if prefix_aware:   # read each shared prompt once per unit of samples
            G = w.num_heads // w.num_kv_heads
            spl, us, ul, mp = B.find_shared_prefixes(w.block_tables, w.context_lens, w.block_size, 16 // G)
            self.sp = {"seq_prefix_len": torch.from_numpy(spl).to(dev), "unit_seqs": torch.from_numpy(us).to(dev),
                       "unit_len": torch.from_numpy(ul).to(dev), "max_prefix_len": mp, "units": len(ul)}
            n = B.shared_prefix_workspace_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.kv_dtype,
                                                w.block_size, w.max_context_len, len(ul), mp, partition_size)
            self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
        self.split = w.max_context_len > self.partition
        torch.cuda.synchronize(dev)
        assert int(self.err.item()) == 0, "setup raised a device error"

    def launches_per_step(self) -> int:
        """Library kernels one step launches: [copy_blocks] + reshape_and_cache + the decode call
        (shared-prefix: [prefix pass] + tail pass + merge; plain: pass 1 + [merge when split])."""
        if self.prefix_aware:
            return ("pairs" in self.d) + 1 + (self.sp["units"] > 0) + 2
        return ("pairs" in self.d) + 1 + 1 + int(self.split)

    def copy_op(self):
        if "pairs" in self.d:
            self.B.copy_blocks(self.k_pool, self.v_pool, self.d["pairs"], device_error=self.err,
                               stream=self.stream)

    def scatter_op(self):
        w = self.w
        self.B.reshape_and_cache(self.d["k_new"], self.d["v_new"], self.k_pool, self.v_pool, self.d["slots"],
                                 float(w.k_scale), float(w.v_scale), device_error=self.err, stream=self.stream)

    def decode_op(self):
        w = self.w
        if self.prefix_aware:
            sp = self.sp
            self.B.paged_attn_decode_shared_prefix(
                self.out, self.d["q"], self.k_pool, self.v_pool, self.d["tables"], self.d["lens"], float(w.scale),
                max_context_len=w.max_context_len, seq_prefix_len=sp["seq_prefix_len"], unit_seqs=sp["unit_seqs"],
                unit_len=sp["unit_len"], max_prefix_len=sp["max_prefix_len"], k_scale=float(w.k_scale),
                v_scale=float(w.v_scale), partition_size=self.partition_arg, workspace=self.ws,
                device_error=self.err, stream=self.stream)
            return
        self.B.paged_attn_decode(self.out, self.d["q"], self.k_pool, self.v_pool, self.d["tables"],
                                 self.d["lens"], float(w.scale), max_context_len=w.max_context_len,
                                 k_scale=float(w.k_scale), v_scale=float(w.v_scale), workspace=self.ws,
                                 partition_size=self.partition_arg, device_error=self.err, stream=self.stream)

    def step(self):
        self.copy_op()
        self.scatter_op()
        self.decode_op()


class PrefillStep:
    """The chunked-prefill workload on one GPU: the cache built, the chunk's inputs resident."""

    def __init__(self, w: wl.PrefillWorkload, dev, kv_fp8: bool = False):
        import torch
        from paged_kv_cache_324_b200 import binding as B
        self.w, self.dev, self.B, self.kv_fp8 = w, dev, B, kv_fp8
        self.stream = torch.cuda.current_stream(dev)
        t16 = {"f16": torch.float16, "bf16": torch.bfloat16}

        def up(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(t16[w.dtype])

        self.k_scale = self.v_scale = 1.0
        if kv_fp8:
            # E4M3 pools with per-tensor amax / 448 scales over everything the step's cache holds
            ops = [op for op in list(w.setup) + [w.step_scatter] if op.slots.size]
            self.k_scale = float(max(wl.amax_scale(op.k, w.dtype) for op in ops))
            self.v_scale = float(max(wl.amax_scale(op.v, w.dtype) for op in ops))
            rng = np.random.default_rng(w.seed + 1)
            n = int(np.prod(w.pool_shape))
            self.k_pool = torch.from_numpy(wl.garbage_bytes(rng, n).reshape(w.pool_shape)).to(dev)
            self.v_pool = torch.from_numpy(wl.garbage_bytes(rng, n).reshape(w.pool_shape)).to(dev)
            self.ws = torch.empty(max(B.prefill_fp8_workspace_bytes(w.num_seqs, w.max_blocks, w.num_kv_heads,
                                                                    w.head_dim, w.block_size), 256),
                                  dtype=torch.uint8, device=dev)
        else:
            self.k_pool, self.v_pool = up(w.initial_pool("k")), up(w.initial_pool("v"))
            # bf16: the workspace V is narrowed into (f16 with a power of two per sequence and KV head)
            need = B.prefill_workspace_bytes(w.dtype, w.num_seqs, w.max_blocks, w.num_kv_heads, w.head_dim,
                                             w.block_size)
            self.ws = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        for op in w.setup:
            if op.slots.size:
                B.reshape_and_cache(up(op.k), up(op.v), self.k_pool, self.v_pool, torch.from_numpy(op.slots).to(dev),
                                    self.k_scale, self.v_scale, device_error=self.err)
        sc = w.step_scatter
        self.host = {"q": w.q, "k_new": sc.k, "v_new": sc.v, "slots": sc.slots, "tables": w.block_tables,
                     "lens": w.context_lens, "qstart": w.query_start}
        self.d = {"q": up(w.q), "k_new": up(sc.k), "v_new": up(sc.v), "slots": torch.from_numpy(sc.slots).to(dev),
                  "tables": torch.from_numpy(w.block_tables).to(dev), "lens": torch.from_numpy(w.context_lens).to(dev),
                  "qstart": torch.from_numpy(w.query_start).to(dev)}
        self.out = torch.empty_like(self.d["q"])
        torch.cuda.synchronize(dev)
        assert int(self.err.item()) == 0, "setup raised a device error"

    def scatter_op(self):
        self.B.reshape_and_cache(self.d["k_new"], self.d["v_new"], self.k_pool, self.v_pool, self.d["slots"],
                                 self.k_scale, self.v_scale, device_error=self.err, stream=self.stream)

    def prefill_op(self):
        w = self.w
        if self.kv_fp8:
            self.B.paged_attn_prefill_fp8(self.out, self.d["q"], self.k_pool, self.v_pool, self.d["tables"],
                                          self.d["lens"], self.d["qstart"], float(w.scale), self.k_scale,
                                          self.v_scale, max_query_len=w.max_query_len, workspace=self.ws,
                                          device_error=self.err, stream=self.stream)
            return
        self.B.paged_attn_prefill(self.out, self.d["q"], self.k_pool, self.v_pool, self.d["tables"], self.d["lens"],
                                  self.d["qstart"], float(w.scale), max_query_len=w.max_query_len,
                                  workspace=self.ws, device_error=self.err, stream=self.stream)

    def step(self):
        self.scatter_op()
        self.prefill_op()


PREFILL_METRIC = "paged prefill attention TFLOP/s (causal chunk over the paged cache)"


def tensor_peak():
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def run_prefill(args, rank, world, local_rank):
    """The chunked-prefill step (scatter of the chunk's K/V, then the prefill) timed like decode."""
    import torch
    dist_on = world > 1
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    kv_fp8 = args.config == "prefill_fp8"
    w = wl.make_prefill()
    ps = PrefillStep(w, dev, kv_fp8)
    flops = wl.prefill_flops(w)
    for _ in range(args.warmup):
        ps.step()
    barrier_sync(torch, dist_on)
    K = args.steps
    # K steps replayed from one CUDA graph, clocks sampled meanwhile
    g = capture(torch, ps, ps.step, K)
    ms_total, clk_report = time_graph(torch, g, dist_on, local_rank)
    del g
    ms_step = max_over_ranks(torch, ms_total, dist_on) / K
    # the prefill call's own rate: K calls back to back from one graph (the roofline's duration),
    # with its own clock record: a back-to-back tensor-core load can meet the power cap sooner
    g = capture(torch, ps, ps.prefill_op, K)
    pf_total, clk_stream = time_graph(torch, g, dist_on, local_rank)
    del g
    pf_stream_ms = max_over_ranks(torch, pf_total, dist_on) / K
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier_sync(torch, dist_on)
    for i in range(K):
        ev[i][0].record()
        ps.scatter_op()
        ev[i][1].record()
        ps.prefill_op()
        ev[i][2].record()
    barrier_sync(torch, dist_on)
    assert int(ps.err.item()) == 0, "device error during the timed region"
    pf_ms = sum(ev[i][1].elapsed_time(ev[i][2]) for i in range(K)) / K
    sc_ms = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)) / K
    total_flops = sum_over_ranks(torch, float(flops), dist_on)
    value = total_flops / (ms_step * 1e-3) / 1e12

    pinned = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16
                                  else np.ascontiguousarray(v)).pin_memory() for k, v in ps.host.items()}
    dq = {k: (ps.d[k].view(torch.int16) if ps.d[k].dtype in (torch.float16, torch.bfloat16) else ps.d[k])
          for k in pinned}
    out_host = torch.empty(ps.out.shape, dtype=ps.out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        for k, v in pinned.items():
            dq[k].copy_(v, non_blocking=True)
        ps.step()
        out_host.copy_(ps.out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    barrier_sync(torch, dist_on)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(K):
        e2e_step()
    e2.record()
    barrier_sync(torch, dist_on)
    e2e_serial_ms = max_over_ranks(torch, s2.elapsed_time(e2), dist_on) / K
    e2e_ms = pipelined_e2e_ms(torch, dev, ps, pinned, args.warmup, K, dist_on)
    peak, peak_sus, kind = tensor_peak()
    achieved = flops / (pf_stream_ms * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": (w.dtype + " q.K^T (E4M3 cache widened exactly: K to " + w.dtype + ", V to f16), f16 P.V, "
                  "f32 accumulate") if kv_fp8
        else (w.dtype + " q.K^T, f16 P.V (V narrowed to f16 per sequence and KV head), f32 accumulate"
              if w.dtype == "bf16" else w.dtype + " operands, f32 accumulate"),
        "data": "synthetic (seeded N(0,1) q/K/V; random-byte pool content in unwritten slots)",
        "config": {"workload": w.description + (", E4M3 cache (per-tensor amax/448 scales)" if kv_fp8 else ""),
                   "name": "prefill_fp8" if kv_fp8 else w.name, "num_seqs": w.num_seqs, "num_tokens": w.num_tokens,
                   "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size, "num_blocks": w.num_blocks,
                   "total_context_tokens": int(w.context_lens.sum()), "flops_per_step": flops,
                   "step": ("reshape_and_cache (the chunk's K/V, quantised to E4M3) + paged_attn_prefill_fp8 "
                            "(widen_blocks_kernel, then paged_prefill_kernel)") if kv_fp8
                   else "reshape_and_cache (the chunk's K/V) + paged_attn_prefill (v_absmax_kernel, "
                        "v_narrow_kernel, then paged_prefill_kernel)",
                   "l2": "no flush: the step reads %.0f MB of K/V and q, %.0f MB of output are written; the "
                         "kernel is bound by the tensor cores, not HBM" % (wl.prefill_bytes(w) / 1e6,
                                                                           w.num_tokens * w.num_heads * w.head_dim * 2 / 1e6),
                   "parallelism": f"dp{world}" if world > 1 else "single GPU"},
        "tokens_per_s": round(sum_over_ranks(torch, float(w.num_tokens), dist_on) / (ms_step * 1e-3), 1),
        "prefill_ms_in_stream": round(pf_stream_ms, 5),
        "kernel_ms": {("paged_attn_prefill_fp8" if kv_fp8 else "paged_attn_prefill"): round(pf_ms, 5),
                      "reshape_and_cache": round(sc_ms, 5)},
        "roofline": {"bound": "tensor",
                     "kernel": ("the paged_attn_prefill_fp8 call (widen_blocks_kernel + paged_prefill_kernel)"
                                if kv_fp8 else "the paged_attn_prefill call (v_absmax_kernel + v_narrow_kernel + "
                                               "paged_prefill_kernel)"),
                     "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "frac_of_sustained": round(achieved / peak_sus, 4),
                     "traffic": (PREFILL_TRAFFIC[args.config]["bytes_per_launch"]
                                 if PREFILL_TRAFFIC[args.config]["kernel_sha"] == prefill_source_sha() else None),
                     "flops_per_launch": flops,
                     "flops_counted": "4 * head_dim * num_heads * causal (query, key) pairs",
                     "peak_kind": f"{kind} (cuBLAS bf16, burst; sustained {peak_sus})"},
        "e2e": {"value": round(total_flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": PIPELINE_NOTE,
                "serial_value": round(total_flops / (e2e_serial_ms * 1e-3) / 1e12, 2),
                "serial_ms_per_step": round(e2e_serial_ms, 5)},
        "gpu_launches": (3 if kv_fp8 else 4) * K,
        "timing": ("value: CUDA events around one replay of a CUDA graph holding K steps; roofline: K prefill "
                   "calls back to back from one graph in the same run (prefill_ms_in_stream, clocks_stream); "
                   "kernel_ms: CUDA events around each call in a third pass"),
        "clocks": clk_report,
        "clocks_stream": clk_stream,
    }
    return line, w


class PrefillOracleRunner:
    """The float64 oracle's prefill on the host's cores, holding the workload's pools (built once)."""

    def __init__(self, w: wl.PrefillWorkload, kv_fp8: bool = False):
        import oracle
        self.o, self.w = oracle, w
        ops = [op for op in list(w.setup) + [w.step_scatter] if op.slots.size]
        if kv_fp8:
            self.kv_dtype = "e4m3"
            self.ks = float(max(wl.amax_scale(op.k, w.dtype) for op in ops))
            self.vs = float(max(wl.amax_scale(op.v, w.dtype) for op in ops))
            rng = np.random.default_rng(w.seed + 1)
            n = int(np.prod(w.pool_shape))
            self.kp = wl.garbage_bytes(rng, n).reshape(w.pool_shape)
            self.vp = wl.garbage_bytes(rng, n).reshape(w.pool_shape)
        else:
            self.kv_dtype, self.ks, self.vs = w.dtype, 1.0, 1.0
            self.kp, self.vp = w.initial_pool("k"), w.initial_pool("v")
        for op in ops:
            oracle.reshape_and_cache(op.k, op.v, w.dtype, self.kp, self.vp, self.kv_dtype, op.slots, self.ks, self.vs)
        self.rng = np.random.default_rng(12)
        self.cores = os.cpu_count() or 1

    def sample(self, budget_s: float, slice_rows: int = 64):
        """Slices of ``slice_rows`` consecutive query rows of random chunks, each over its full
        causal prefix, until the budget is spent (at least one); returns (rows, flops, seconds)."""
        w, o = self.w, self.o
        rows, flops, t0 = 0, 0, time.perf_counter()
        while True:
            s = int(self.rng.integers(0, w.num_seqs))
            q0, q1 = int(w.query_start[s]), int(w.query_start[s + 1])
            n = min(slice_rows, q1 - q0)
            r0 = int(self.rng.integers(q0, q1 - n + 1))
            L = int(w.context_lens[s]) - (q1 - q0) + (r0 - q0) + n
            o.paged_attn_prefill(w.q[r0:r0 + n], w.dtype, self.kp, self.vp, self.kv_dtype, w.block_tables[s:s + 1],
                                 np.array([L], np.int32), np.array([0, n], np.int32), w.scale, self.ks, self.vs,
                                 threads=self.cores)
            rows += n
            flops += 4 * w.head_dim * w.num_heads * (n * (L - n) + n * (n + 1) // 2)
            el = time.perf_counter() - t0
            if el >= budget_s:
                return rows, flops, el


SWAP_METRIC = "block swap GB/s over the host link (GPU pool <-> pinned host pool, both directions)"


def run_swap(args, rank, world, local_rank):
    """Preemption by swapping: each step moves a group's blocks GPU -> pinned host (pkv_swap_blocks)
    and another group's blocks host -> GPU.  Pools of the OPT-13B layer shape."""
    import torch
    from paged_kv_cache_324_b200 import binding as B
    dist_on = world > 1
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    NB, NH, Hkv, Bs, D, n = 16384, 4096, 40, 16, 128, 1024     # 1024 blocks = 16 sequences of 1,024 tokens
    rng = np.random.default_rng(7)
    torch.manual_seed(7)
    kp = torch.empty((NB, Hkv, Bs, D), dtype=torch.float16, device=dev).normal_()
    vp = torch.empty_like(kp).normal_()
    hk = torch.empty((NH, Hkv, Bs, D), dtype=torch.float16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    block_bytes = Hkv * Bs * D * 2
    out_pairs = np.stack([rng.choice(NB, n, replace=False), rng.choice(NH // 2, n, replace=False)], axis=1)
    in_pairs = np.stack([NH // 2 + rng.choice(NH // 2, n, replace=False), rng.choice(NB, n, replace=False)], axis=1)
    host_pairs = {"out": out_pairs.astype(np.int64), "in": in_pairs.astype(np.int64)}
    dpairs = {k: torch.from_numpy(v).to(dev) for k, v in host_pairs.items()}
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    step_bytes = 2 * 2 * n * block_bytes                         # K and V, out and in

    def step():
        B.swap_blocks(kp, vp, hk, hv, dpairs["out"], device_error=err)
        B.swap_blocks(hk, hv, kp, vp, dpairs["in"], device_error=err)

    for _ in range(args.warmup):
        step()
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier_sync(torch, dist_on)
        start.record()
        for _ in range(K):
            step()
        end.record()
        barrier_sync(torch, dist_on)
    ms_step = max_over_ranks(torch, start.elapsed_time(end), dist_on) / K
    assert int(err.item()) == 0, "device error during the timed region"
    # per direction, and the copy engines' rate for the same bytes (the link's measured peak here)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    for _ in range(K):
        B.swap_blocks(kp, vp, hk, hv, dpairs["out"], device_error=err)
    ev[1].record()
    for _ in range(K):
        B.swap_blocks(hk, hv, kp, vp, dpairs["in"], device_error=err)
    ev[2].record()
    torch.cuda.synchronize()
    out_ms, in_ms = ev[0].elapsed_time(ev[1]) / K, ev[1].elapsed_time(ev[2]) / K
    nbytes = n * block_bytes
    big_d, big_h = torch.empty(nbytes, dtype=torch.uint8, device=dev), torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    ce = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(2):
        big_h.copy_(big_d, non_blocking=True)
        big_d.copy_(big_h, non_blocking=True)
    ce[0].record()
    for _ in range(4):
        big_h.copy_(big_d, non_blocking=True)
    ce[1].record()
    for _ in range(4):
        big_d.copy_(big_h, non_blocking=True)
    ce[2].record()
    torch.cuda.synchronize()
    d2h = nbytes / (ce[0].elapsed_time(ce[1]) / 4 * 1e-3) / 1e9
    h2d = nbytes / (ce[1].elapsed_time(ce[2]) / 4 * 1e-3) / 1e9
    peak = step_bytes / ((step_bytes / 2) / (d2h * 1e9) + (step_bytes / 2) / (h2d * 1e9)) / 1e9
    value = sum_over_ranks(torch, float(step_bytes), dist_on) / (ms_step * 1e-3) / 1e9
    achieved = step_bytes / (ms_step * 1e-3) / 1e9
    # end to end: the step's pairs come from pinned host memory each step
    pin = {k: torch.from_numpy(v).pin_memory() for k, v in host_pairs.items()}
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(K):
        for k in pin:
            dpairs[k].copy_(pin[k], non_blocking=True)
        step()
        err_h = err.to("cpu", non_blocking=True)
    e2.record()
    barrier_sync(torch, dist_on)
    e2e_ms = max_over_ranks(torch, s2.elapsed_time(e2), dist_on) / K
    line = {
        "metric": SWAP_METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 (bytes moved as is)",
        "data": "synthetic (N(0,1) pools; random distinct block pairs)",
        "config": {"workload": f"swap out {n} blocks GPU -> pinned host and {n} blocks host -> GPU per step; "
                               f"pools [{NB} | {NH}, {Hkv}, {Bs}, {D}] f16 (OPT-13B layer shape)",
                   "name": "swap", "blocks_per_direction": n, "block_bytes_per_pool": block_bytes,
                   "step": "pkv_swap_blocks (out) + pkv_swap_blocks (in)",
                   "l2": "no flush: each step moves %.0f MB, more than the 126 MB L2" % (step_bytes / 1e6),
                   "parallelism": f"dp{world}" if world > 1 else "single GPU"},
        "kernel_ms": {"swap_out": round(out_ms, 5), "swap_in": round(in_ms, 5)},
        "roofline": {"bound": "link", "kernel": "swap_blocks_kernel", "achieved": round(achieved, 2),
                     "peak": round(peak, 2), "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "bytes_per_step": step_bytes,
                     "peak_kind": f"measured in this run: copy engines on one {nbytes >> 20} MiB pinned buffer, "
                                  f"device->host {d2h:.1f} GB/s, host->device {h2d:.1f} GB/s, combined for "
                                  f"equal bytes each way",
                     "per_direction_gbs": {"out": round(nbytes * 2 / (out_ms * 1e-3) / 1e9, 2),
                                           "in": round(nbytes * 2 / (in_ms * 1e-3) / 1e9, 2)}},
        "e2e": {"value": round(step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(e2e_ms, 5),
                "h2d_bytes_per_step": sum(v.nbytes for v in host_pairs.values()), "d2h_bytes_per_step": 4},
        "gpu_launches": 2 * K,
        "timing": "value: CUDA events around K back-to-back steps",
        "clocks": clk.report(),
    }
    return line


def pipelined_e2e_ms(torch, dev, step_obj, pinned, warmup, K, dist_on) -> float:
    """Milliseconds per step of the end-to-end loop as a serving engine runs it: two sets of input
    and output buffers and one copy stream per direction, so that step i+1's inputs cross the
    link while step i computes and step i-1's output comes back.  Every step still copies all of
    its inputs in (from the pinned host tensors in `pinned`) and its output back.  `step_obj`
    has `d` (device inputs by the same keys), `out`, `stream` and `step()`."""
    import copy as _copy
    second = _copy.copy(step_obj)
    second.d = {k: v.clone() for k, v in step_obj.d.items()}
    second.out = torch.empty_like(step_obj.out)
    sets = [step_obj, second]

    def as_bits(t):
        return t.view(torch.int16) if t.dtype in (torch.float16, torch.bfloat16) else t

    dst = [{k: as_bits(x.d[k]) for k in pinned} for x in sets]
    out_host = [torch.empty(step_obj.out.shape, dtype=step_obj.out.dtype).pin_memory() for _ in sets]
    comp, s_in, s_out = step_obj.stream, torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_ready = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_free[b])             # the set's previous step and read-back are done
                for k, v in pinned.items():
                    dst[b][k].copy_(v, non_blocking=True)
                ev_ready[b].record(s_in)
            comp.wait_event(ev_ready[b])
            sets[b].step()
            ev_done[b].record(comp)
            with torch.cuda.stream(s_out):                  # a read-back must not hold up the next inputs
                s_out.wait_event(ev_done[b])
                out_host[b].copy_(sets[b].out, non_blocking=True)
                ev_free[b].record(s_out)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)

    run(max(warmup, 2))
    barrier_sync(torch, dist_on)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    s_in.wait_event(s)
    s_out.wait_event(s)
    run(K)
    e.record(comp)
    barrier_sync(torch, dist_on)
    return max_over_ranks(torch, s.elapsed_time(e), dist_on) / K


PIPELINE_NOTE = ("two buffer sets and one copy stream per direction: step i+1's inputs are copied in, and "
                 "step i-1's output copied back, while step i computes")


def barrier_sync(torch, dist_on):
    if dist_on:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(torch, x: float, dist_on: bool, device: str = "cuda") -> float:
    """Slowest rank's time: the job's time under weak scaling."""
    if not dist_on:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(torch, x: float, dist_on: bool, device: str = "cuda") -> float:
    """Whole-job quantity (bytes, sequences) summed over ranks."""
    if not dist_on:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(step_bytes_this_rank: float, ms_total_this_rank: float, steps: int, dist_on: bool,
                   torch, device: str = "cuda"):
    """(GB/s of the whole job, ms per step): bytes of all ranks / the slowest rank's time."""
    ms_step = max_over_ranks(torch, ms_total_this_rank, dist_on, device) / steps
    total = sum_over_ranks(torch, float(step_bytes_this_rank), dist_on, device)
    return total / (ms_step * 1e-3) / 1e9, ms_step


def capture(torch, ds, fn, K: int):
    """One CUDA graph of K calls of fn() (the library's launches on a capturing side stream), as a
    serving loop replays a step; the kernels keep their programmatic-dependent-launch edges."""
    side = torch.cuda.Stream(ds.dev)
    side.wait_stream(torch.cuda.current_stream(ds.dev))
    saved = ds.stream
    ds.stream = side
    try:
        with torch.cuda.stream(side):
            fn()                                   # one eager call on the side stream before capture
        torch.cuda.current_stream(ds.dev).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for _ in range(K):
                fn()
    finally:
        ds.stream = saved
    torch.cuda.synchronize(ds.dev)
    return g


def time_graph(torch, g, dist_on: bool, local_rank: int = None):
    """Device time (ms) of one replay, CUDA events on the stream the replay is launched on, with the
    clocks sampled meanwhile when local_rank is given: (ms, clocks or None)."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()                                     # warm: the graph's first launch uploads it
    barrier_sync(torch, dist_on)
    clk = ClockSampler(local_rank) if local_rank is not None else None
    if clk:
        clk.__enter__()
    try:
        barrier_sync(torch, dist_on)
        start.record()
        g.replay()
        end.record()
        barrier_sync(torch, dist_on)
    finally:
        if clk:
            clk.__exit__(None, None, None)
    return start.elapsed_time(end), (clk.report() if clk else None)


def time_steps(torch, ds, K: int, dist_on: bool, local_rank: int):
    """Device time of K steps replayed from one CUDA graph (no host launch cost between kernels, and
    no events between them, so they overlap as a serving loop's do), with the clocks sampled
    meanwhile: (ms in total, clocks)."""
    g = capture(torch, ds, ds.step, K)
    ms, clocks = time_graph(torch, g, dist_on, local_rank)
    del g
    return ms, clocks


def time_steps_eager(torch, ds, K: int, dist_on: bool) -> float:
    """The same K steps launched one by one from Python (ms in total, max over ranks)."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier_sync(torch, dist_on)
    start.record()
    for _ in range(K):
        ds.step()
    end.record()
    barrier_sync(torch, dist_on)
    return max_over_ranks(torch, start.elapsed_time(end), dist_on)


def time_decode_stream(torch, ds, K: int, dist_on: bool) -> float:
    """Milliseconds per decode call over K calls back to back, replayed from one CUDA graph (events
    only at both ends): the dominant kernel's own rate, never more than the step that contains
    it, since each step runs the same call plus the scatter (and copies)."""
    g = capture(torch, ds, ds.decode_op, K)
    ms, _ = time_graph(torch, g, dist_on)
    del g
    return max_over_ranks(torch, ms, dist_on) / K


def time_each_call(torch, ds, K: int, dist_on: bool) -> dict:
    """Mean milliseconds of each call with CUDA events around every call (these events keep
    the kernels from overlapping, so the per-call times add up to more than a step)."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    barrier_sync(torch, dist_on)
    for i in range(K):
        e = ev[i]
        e[0].record()
        ds.copy_op()
        e[1].record()
        ds.scatter_op()
        e[2].record()
        ds.decode_op()
        e[3].record()
    barrier_sync(torch, dist_on)
    mean = lambda a, b: sum(ev[i][a].elapsed_time(ev[i][b]) for i in range(K)) / K  # noqa: E731
    return {"paged_attn_decode": round(mean(2, 3), 5), "reshape_and_cache": round(mean(1, 2), 5),
            "copy_blocks": round(mean(0, 1), 5) if "pairs" in ds.d else None}


def read_peak(torch, ds, reps: int = 5) -> float:
    """Read-only HBM rate (GB/s) of a pass over this workload's K and V pools (pkv_stream_read),
    timed with CUDA events on the launching stream: the denominator for a read-mostly kernel."""
    from paged_kv_cache_324_b200 import binding as B
    sink = torch.zeros(1, dtype=torch.int32, device=ds.k_pool.device)
    pools = (ds.k_pool.view(torch.uint8).view(-1), ds.v_pool.view(torch.uint8).view(-1))
    nbytes = sum(p.numel() for p in pools)
    for _ in range(2):
        for p in pools:
            B.stream_read(p, sink)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(reps):
        for p in pools:
            B.stream_read(p, sink)
    e.record()
    torch.cuda.synchronize()
    return nbytes * reps / (s.elapsed_time(e) * 1e-3) / 1e9, nbytes


def traffic_for(name: str, partition_arg: str, prefix_aware: bool, heads: bool):
    """ncu DRAM bytes of one decode call, if a capture of this exact kernel source exists."""
    tr = NCU_TRAFFIC.get(name)
    # the capture ran the plain decode at the workload's own partition size
    if tr and tr.get("kernel_sha") == decode_source_sha() and partition_arg == "config" and not prefix_aware \
            and not heads:
        return tr["bytes_per_launch"]
    return None


def measure_decode(torch, w, dev, ps: int, prefix_aware: bool, K: int, warmup: int, dist_on: bool,
                   local_rank: int, peak: float, peak_kind: str, rpeak: float, partition_arg: str = "config",
                   heads: bool = False):
    """One decode workload on this GPU: the step rate, the decode call's roofline, per-call times.
    Returns (result dict, DeviceStep)."""
    ds = DeviceStep(w, dev, ps, prefix_aware=prefix_aware)
    step_bytes = wl.step_algorithmic_bytes(w)
    # the roofline counts each physical KV slot once: on shared prompts that is what must cross HBM
    roof_bytes = wl.decode_distinct_bytes(w)
    for _ in range(warmup):
        ds.step()
    barrier_sync(torch, dist_on)
    ms_total, clocks = time_steps(torch, ds, K, dist_on, local_rank)
    eager_ms = time_steps_eager(torch, ds, K, dist_on) / K
    dec_ms = time_decode_stream(torch, ds, K, dist_on)
    kernel_ms = time_each_call(torch, ds, K, dist_on)
    assert int(ds.err.item()) == 0, "device error during the timed region"
    value, ms_step = job_throughput(step_bytes, ms_total, K, dist_on, torch)
    achieved = roof_bytes / (dec_ms * 1e-3) / 1e9
    res = {
        "value": round(value, 2), "ms_per_step": round(ms_step, 5), "eager_ms_per_step": round(eager_ms, 5),
        "sequences_per_s": round(sum_over_ranks(torch, float(w.num_seqs), dist_on) / (ms_step * 1e-3), 1),
        "decode_ms_in_stream": round(dec_ms, 5), "kernel_ms": kernel_ms,
        "roofline": {"bound": "hbm", "kernel": "paged_decode_kernel + decode_reduce_kernel",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_read": round(rpeak, 1), "frac_read": round(achieved / rpeak, 4),
                     "traffic": traffic_for(w.name, partition_arg, prefix_aware, heads),
                     "bytes_per_launch": roof_bytes,
                     "bytes_counted": "distinct KV slots attended (each once) + q + out + table entries + lengths",
                     "peak_kind": f"{peak_kind} (copy, burst)",
                     "peak_read_kind": "measured in this run (pkv_stream_read over the K and V pools)",
                     "duration": "decode_ms_in_stream: K decode calls back to back from one CUDA graph, CUDA "
                                 "events at both ends"},
        "clocks": clocks,
    }
    return res, ds


def config_summary(w, ds) -> dict:
    plan = "plain"
    if ds.prefix_aware:
        plan = ds.B.shared_prefix_plan_used(ds.sp["units"], w.num_kv_heads, w.head_dim, w.kv_dtype,
                                            ds.sp["max_prefix_len"])
    return {"workload": w.description, "name": w.name, "num_seqs": w.num_seqs, "num_heads": w.num_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "num_blocks": w.num_blocks, "max_context_len": w.max_context_len,
            "total_context_tokens": int(w.context_lens.sum()), "partition_size": ds.partition,
            "partition_rule": "automatic" if ds.partition_arg == 0 else "set by the workload or --partition",
            "kv_dtype": w.kv_dtype,
            "step": ("copy_blocks + " if "pairs" in ds.d else "") + "reshape_and_cache + " +
                    ("paged_attn_decode_shared_prefix (plan: %s)" % plan if ds.prefix_aware else "paged_attn_decode"),
            "step_bytes": wl.step_algorithmic_bytes(w), "decode_bytes": wl.decode_algorithmic_bytes(w),
            "decode_distinct_bytes": wl.decode_distinct_bytes(w)}


def l2_note(roof_bytes: int) -> str:
    if roof_bytes > L2_BYTES:
        return "no flush: each step reads %.2f GB of distinct KV, more than the 126 MB L2" % (roof_bytes / 1e9)
    return ("no flush: the %.0f MB of distinct KV fit in the 126 MB L2, so repeated reads of shared blocks may "
            "hit L2" % (roof_bytes / 1e6))


#: the other decode workloads measured in the default run (name, shared-prefix call)
CONFIG_ROWS = [("gqa", False), ("fp8", False), ("fp8_b32", False), ("prefix", False), ("prefix", True),
               ("prefix_long", False), ("prefix_long", True)]


def run_configs(args, torch, dev, dist_on, local_rank, peak, peak_kind, rpeak) -> dict:
    """Every workload of CONFIG_ROWS, timed like the headline (K steps back to back, then the decode
    call's stream), one after the other with the previous one's memory released."""
    out = {}
    for name, shared in CONFIG_ROWS:
        w = wl.make(name)
        ps = w.partition_size if args.partition == "config" else (0 if args.partition == "auto"
                                                                  else int(args.partition))
        res, ds = measure_decode(torch, w, dev, ps, shared, args.steps, args.warmup, dist_on, local_rank, peak,
                                 peak_kind, rpeak, args.partition)
        key = name + ("+shared_prefix_call" if shared else "")
        res["config"] = config_summary(w, ds)
        res["config"]["l2"] = l2_note(wl.decode_distinct_bytes(w))
        res["gpu_launches"] = ds.launches_per_step() * args.steps
        out[key] = res
        del ds
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    dist_on = world > 1
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = wl.make(args.config)        # weak scaling: every rank runs a batch of the same shape
    heads = args.shard == "heads" and world > 1
    if heads:                       # strong scaling: one batch, each rank its share of the KV heads
        w = wl.shard_heads(w, rank, world)
    ps = w.partition_size if args.partition == "config" else (0 if args.partition == "auto" else int(args.partition))
    peak, peak_kind = hbm_peak()
    K = args.steps
    # the read-only denominator first, on this workload's pools (each rank its own)
    probe = DeviceStep(w, dev, ps, prefix_aware=args.prefix_aware)
    rpeak, rbytes = read_peak(torch, probe)
    del probe
    torch.cuda.empty_cache()
    res, ds = measure_decode(torch, w, dev, ps, args.prefix_aware, K, args.warmup, dist_on, local_rank, peak,
                             peak_kind, rpeak, args.partition, heads)
    step_bytes = wl.step_algorithmic_bytes(w)
    total_bytes = sum_over_ranks(torch, float(step_bytes), dist_on)
    ms_step = res["ms_per_step"]

    # end to end: the step's inputs from pinned host memory, the output back to the host
    def pin(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).pin_memory()

    pinned = {k: pin(v) for k, v in ds.host.items()}
    dq = {k: (ds.d[k].view(torch.int16) if ds.d[k].dtype in (torch.float16, torch.bfloat16) else ds.d[k])
          for k in pinned}
    out_host = torch.empty(ds.out.shape, dtype=ds.out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        for k, v in pinned.items():
            dq[k].copy_(v, non_blocking=True)
        ds.step()
        out_host.copy_(ds.out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    barrier_sync(torch, dist_on)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(K):
        e2e_step()
    e2.record()
    barrier_sync(torch, dist_on)
    e2e_serial_ms = max_over_ranks(torch, s2.elapsed_time(e2), dist_on) / K

    # the same, pipelined as a serving loop runs it
    e2e_ms = pipelined_e2e_ms(torch, dev, ds, pinned, args.warmup, K, dist_on)
    e2e_value = total_bytes / (e2e_ms * 1e-3) / 1e9
    e2e_serial_value = total_bytes / (e2e_serial_ms * 1e-3) / 1e9
    cfg = config_summary(w, ds)
    cfg["l2"] = l2_note(wl.decode_distinct_bytes(w))
    cfg["parallelism"] = (f"tp{world} (KV heads split, identical block tables)" if heads
                          else f"dp{world}" if world > 1 else "single GPU")
    roof = res["roofline"]
    roof["peak_read_bytes"] = rbytes
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if heads else "weak", "vs_baseline": None,
        "dtype": w.kv_dtype if w.kv_dtype != "e4m3" else "e4m3 (KV), f16 (q/out), f32 accumulate",
        "data": "synthetic (seeded N(0,1) K/V/q; random-byte pool content in unwritten slots)",
        "config": cfg,
        "sequences_per_s": round((w.num_seqs if heads else sum_over_ranks(torch, float(w.num_seqs), dist_on))
                                 / (ms_step * 1e-3), 1),
        "pct_of_hbm_peak": round(100 * res["value"] / world / peak, 2),
        "pct_of_nominal_8tbs": round(100 * res["value"] / world / NOMINAL_HBM_GBS, 2),
        "eager_ms_per_step": res["eager_ms_per_step"],
        "decode_ms_in_stream": res["decode_ms_in_stream"],
        "kernel_ms": res["kernel_ms"],
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "ms_per_step": round(e2e_ms, 5),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": PIPELINE_NOTE,
                "serial_value": round(e2e_serial_value, 2), "serial_ms_per_step": round(e2e_serial_ms, 5)},
        "gpu_launches": ds.launches_per_step() * K,
        "timing": ("value and ms_per_step: CUDA events around one replay of a CUDA graph holding K steps (as a "
                   "serving loop replays its step; eager_ms_per_step: the same K steps launched one by one from "
                   "Python); roofline: K decode calls back to back from one graph in the same run "
                   "(decode_ms_in_stream); kernel_ms: CUDA events around each call in a further pass (events "
                   "between kernels stop their overlap, so those add up to more than a step)"),
        "clocks": res["clocks"],
    }
    del ds, pinned, dq
    torch.cuda.empty_cache()
    if world == 1 and not args.no_configs:
        line["configs"] = run_configs(args, torch, dev, dist_on, local_rank, peak, peak_kind, rpeak)
    return line, w


class OracleRunner:
    """The float64 oracle on the host's cores, holding the workload's pools."""

    def __init__(self, w: wl.DecodeWorkload):
        import oracle
        self.o, self.w = oracle, w
        self.kp, self.vp = w.initial_pool("k"), w.initial_pool("v")
        for op in w.setup:
            if isinstance(op, wl.Scatter):
                oracle.reshape_and_cache(op.k, op.v, w.src_dtype, self.kp, self.vp, w.kv_dtype, op.slots,
                                         w.k_scale, w.v_scale)
            else:
                oracle.copy_blocks(self.kp, self.vp, op.pairs)
        self.cores = os.cpu_count() or 1

    def step(self, n=None) -> int:
        """One step on the first n sequences (all by default); returns its algorithmic bytes."""
        o, w = self.o, self.w
        n = w.num_seqs if n is None else n
        b = 0
        if w.step_copy is not None:
            o.copy_blocks(self.kp, self.vp, w.step_copy.pairs)
            b += wl.copy_algorithmic_bytes(w, w.step_copy)
        sc = w.step_scatter
        o.reshape_and_cache(sc.k[:n], sc.v[:n], w.src_dtype, self.kp, self.vp, w.kv_dtype, sc.slots[:n],
                            w.k_scale, w.v_scale)
        o.paged_attn_decode(w.q[:n], w.q_dtype, self.kp, self.vp, w.kv_dtype, w.block_tables[:n],
                            w.context_lens[:n], w.scale, w.k_scale, w.v_scale, threads=self.cores)
        sub = wl.Scatter(sc.k[:n], sc.v[:n], sc.slots[:n])
        lens = w.context_lens[:n].astype(np.int64)
        b += wl.scatter_algorithmic_bytes(w, sub)
        b += int(lens.sum()) * wl.kv_bytes_per_token(1, w.num_kv_heads, w.head_dim, wl.ELEM_BYTES[w.kv_dtype])
        b += 2 * n * w.num_heads * w.head_dim * wl.ELEM_BYTES[w.q_dtype]
        b += 4 * int(((lens + w.block_size - 1) // w.block_size).sum()) + 4 * n
        return b


def cpu_oracle_sample(w: wl.DecodeWorkload, budget_s: float, one_core_s: float = 3.0):
    """Whole steps of the workload on the oracle (all host cores) until the budget is spent (at
    least one); then, on one core, a step over the first sequences, as many as fit in about
    ``one_core_s`` after a one-sequence calibration.  Returns (steps, bytes, seconds, cores,
    (one-core sequences, bytes, seconds))."""
    r = OracleRunner(w)
    n, nbytes, t0 = 0, 0, time.perf_counter()
    while True:
        nbytes += r.step()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    cores, r.cores = r.cores, 1
    t1 = time.perf_counter()
    r.step(1)
    t1 = time.perf_counter() - t1
    n1 = max(1, min(w.num_seqs, int(one_core_s / max(t1, 1e-6))))
    t2 = time.perf_counter()
    b1 = r.step(n1)
    el1 = time.perf_counter() - t2
    r.cores = cores
    return n, nbytes, el, cores, (n1, b1, el1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="opt13b",
                    choices=list(wl.NAMES) + list(wl.EXTRA_NAMES) + list(wl.COMPACT_NAMES)
                    + ["prefill", "prefill_fp8", "swap"],
                    help="a decode workload, 'prefill' / 'prefill_fp8' (chunked prefill over a 16-bit or an "
                         "E4M3 cache, TFLOP/s) or 'swap' (block swap, GB/s)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefix-aware", action="store_true",
                    help="decode with pkv_paged_attn_decode_shared_prefix (shared prompts read once per unit)")
    ap.add_argument("--partition", default="config",
                    help="'config' (the workload's stated partition size, else automatic), 'auto', or tokens")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-configs", action="store_true",
                    help="decode workloads: time only --config (by default a single-GPU run also times the "
                         "other decode workloads and reports them under 'configs')")
    ap.add_argument("--shard", default="sequences", choices=["sequences", "heads"],
                    help="decode under torchrun: each rank its own batch (weak scaling) or one batch with the "
                         "KV heads split over the ranks (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference" and args.config == "swap":
        if rank != 0:
            return
        # the oracle's block swap (memcpy per block) between two host pools of the same shape
        import oracle
        NB, NH, Hkv, Bs, D, n = 16384, 4096, 40, 16, 128, 1024
        rng = np.random.default_rng(7)
        gk = np.zeros((NB, Hkv, Bs, D), np.uint16)
        gv = np.zeros_like(gk)
        hk = np.zeros((NH, Hkv, Bs, D), np.uint16)
        hv = np.zeros_like(hk)
        out_p = np.stack([rng.choice(NB, n, replace=False), rng.choice(NH // 2, n, replace=False)], axis=1)
        in_p = np.stack([NH // 2 + rng.choice(NH // 2, n, replace=False), rng.choice(NB, n, replace=False)], axis=1)
        step_bytes = 2 * 2 * n * gk[0].nbytes
        times = []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            oracle.swap_blocks(gk, gv, hk, hv, out_p)
            oracle.swap_blocks(hk, hv, gk, gv, in_p)
            if i >= args.warmup:
                times.append(time.perf_counter() - t0)
        value = step_bytes / (sum(times) / len(times)) / 1e9
        line = {"metric": SWAP_METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * sum(times) / len(times), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "impl": "reference",
                "dtype": "bytes", "data": "synthetic", "config": {"workload": "swap", "name": "swap"},
                "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                                 "sample": f"the whole step (memcpy per block, host memory only), {len(times)} steps"},
                "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if args.impl == "reference" and args.config in ("prefill", "prefill_fp8"):
        if rank != 0:
            return
        w = wl.make_prefill()
        kv_fp8 = args.config == "prefill_fp8"
        r = PrefillOracleRunner(w, kv_fp8)
        cores = r.cores
        per_step = min(30.0, 150.0 / (args.steps + args.warmup))
        slice_rows = 64 if per_step >= 5.0 else 1      # one row over ~2k keys takes tens of ms
        rates, times = [], []
        for i in range(args.warmup + args.steps):
            rows, flops, el = r.sample(per_step, slice_rows)
            if i >= args.warmup:
                rates.append(flops / el)
                times.append(el)
        value = sum(rates) / len(rates) / 1e12
        sample = (f"{slice_rows}-row slices of random chunks (float64 prefill, each row over its full causal "
                  f"prefix{', E4M3 cache' if kv_fp8 else ''}), ~{per_step:.2f} s per step, {len(times)} timed steps")
        line = {"metric": PREFILL_METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * sum(times) / len(times), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "impl": "reference",
                "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.description + (", E4M3 cache (per-tensor amax/448 scales)" if kv_fp8 else ""),
                           "name": args.config},
                "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        w = wl.make(args.config)
        r = OracleRunner(w)
        t0 = time.perf_counter()
        r.step()                                          # calibration: one whole step, untimed
        t_full = time.perf_counter() - t0
        per_step_budget = min(30.0, 150.0 / (args.steps + args.warmup))
        n = max(1, min(w.num_seqs, int(w.num_seqs * per_step_budget / max(t_full, 1e-9))))
        rates, times = [], []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            nbytes = r.step(n)
            el = time.perf_counter() - t0
            if i >= args.warmup:
                rates.append(nbytes / el)
                times.append(el)
        value = sum(rates) / len(rates) / 1e9
        ms = 1e3 * sum(times) / len(times)
        sample = (f"first {n} of {w.num_seqs} sequences per step (scatter + float64 decode), "
                  f"{len(times)} timed steps")
        line = {"metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "impl": "reference",
                "dtype": "f64", "data": "synthetic", "config": {"workload": w.description, "name": w.name},
                "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": r.cores, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    dist_on = world > 1
    if dist_on:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.config == "swap":
            line = run_swap(args, rank, world, local_rank)
            if rank == 0 and world == 1:
                import oracle
                n, NB, NH = 1024, 16384, 4096
                gk = np.zeros((NB, 40, 16, 128), np.uint16)
                hk = np.zeros((NH, 40, 16, 128), np.uint16)
                rng = np.random.default_rng(7)
                pairs = np.stack([rng.choice(NB, n, replace=False), rng.choice(NH, n, replace=False)], axis=1)
                t0, steps = time.perf_counter(), 0
                while time.perf_counter() - t0 < max(args.cpu_budget, 0.5) or steps == 0:
                    oracle.swap_blocks(gk, gk, hk, hk, pairs)
                    oracle.swap_blocks(hk, hk, gk, gk, pairs[:, ::-1])
                    steps += 1
                el = time.perf_counter() - t0
                line["cpu_baseline"] = {"value": round(steps * 2 * 2 * n * gk[0].nbytes / el / 1e9, 3), "unit": "GB/s",
                                        "cores": 1, "kind": "oracle",
                                        "sample": f"{steps} whole step(s) between two host pools (memcpy per block), "
                                                  f"{el:.1f} s"}
            if rank == 0:
                print(json.dumps(line), flush=True)
            return
        if args.config in ("prefill", "prefill_fp8"):
            line, w = run_prefill(args, rank, world, local_rank)
            if rank == 0 and world == 1:
                r = PrefillOracleRunner(w, args.config == "prefill_fp8")
                rows, flops, el = r.sample(args.cpu_budget)
                line["cpu_baseline"] = {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": r.cores,
                                        "kind": "oracle",
                                        "sample": f"{rows} query rows (64-row slices of random chunks, each over "
                                                  f"its full causal prefix, float64), {el:.1f} s"}
            if rank == 0:
                print(json.dumps(line), flush=True)
            return
        line, w = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1:
            n, nbytes, el, cores, (n1, b1, el1) = cpu_oracle_sample(w, args.cpu_budget,
                                                                     one_core_s=min(3.0, args.cpu_budget))
            v = nbytes / el / 1e9
            line["cpu_baseline"] = {"value": round(v, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                                    "sample": f"{n} whole step(s) of the same workload (scatter + float64 decode "
                                              f"of all {w.num_seqs} sequences), {el:.1f} s",
                                    "one_core": {"value": round(b1 / el1 / 1e9, 4), "unit": UNIT, "cores": 1,
                                                 "sample": f"one step over the first {n1} of {w.num_seqs} "
                                                           f"sequences on one thread, {el1:.1f} s"}}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist_on:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
