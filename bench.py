#!/usr/bin/env python
"""Benchmark of the layer-routed hybrid attention hot path on B200.

Default run (the headline): the 256K-context Qwen3-8B-shaped layer pair.
One step = one pass of the whole hot path over one batch of the workload:
  * the CSR of the block pattern (fa_blocksparse_index),
  * two routed layers (fa_hybrid_layer: router pool -> MLP -> argmax on the
    device, then the attention kernel reading the mode): the router head bias
    sends one layer to FULL and one to SPARSE, as in a half-sparse stack,
  * one decode token per layer in that layer's mode (fa_attn_decode).
value = algorithmic FLOPs of the step / time: full layer 4*D*Hq*B*S(S+1)/2,
sparse layer 4*D*Hq*B*(exact attended pairs), decode 4*D*Hq*B*(keys read).
The same line carries the 36-layer hybrid-vs-full projection, the 32-layer
decode step in HBM GB/s ("decode") and the 8K-context layer's kernels
("qwen3-4b-layer-s8192").

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload NAME] [--dry-run]
Multi-GPU: every rank runs an independent replica of the step on its own GPU
(the path has no exchange step); value = all ranks' FLOPs / the slowest
rank's time.  `--gpus N` outside torchrun starts the N ranks itself.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attn TFLOP/s & % bf16 peak; decode HBM GB/s; hybrid vs full at 256K"
DEFAULT_WORKLOAD = "qwen3-8b-layer-s262144"       # 256K prefill, one layer per mode
DECODE_WORKLOAD = "decode-b8-l131072-32l"          # 32-layer decode step
LAYER8K_WORKLOAD = "qwen3-4b-layer-s8192"          # Qwen3-4B layer at 8K
N_INPUT_SETS = 4           # rotated so each step reads inputs not resident in L2
CSRC = os.path.join(ROOT, "block_sparse_attention_layerrouter_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "prefill2_kernel_full_dram_traffic.txt")


# ------------------------------------------------------------ accounting
def flops_full(wl) -> float:
    return 4.0 * 128 * wl.Hq * wl.B * (wl.S * (wl.S + 1) / 2)


def flops_sparse_exact(wl) -> float:
    import oracle  # pair counting only (host arithmetic of the pattern)
    return 4.0 * 128 * wl.Hq * wl.B * oracle.attended_pairs_sparse(wl.S, 64, wl.sink, wl.window)


def csr_nnz(S, sink, window) -> int:
    nb = -(-S // 64)
    sb, wb = sink // 64, window // 64
    n = 0
    for i in range(nb):
        a = min(sb, i + 1)
        lo = max(a, i - wb + 1)
        n += a + (i - lo + 1)
    return n


def decode_keys(L, mode, sink, window) -> int:
    if mode == 0:
        return L
    last = (L - 1) // 64
    a = min(sink // 64, last + 1)
    lo = max(a, last - window // 64 + 1)
    keys = a * 64
    for blk in range(lo, last + 1):
        keys += min(L, (blk + 1) * 64) - blk * 64
    return keys


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""

    def __init__(self, device: torch.device, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(device)
            bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self._nvml = None
            self.error = str(e)

    _NAMES = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
              0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
              0x100: "display_clocks", 0x1: "gpu_idle", 0x10: "sync_boost"}

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self._NAMES.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self._period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def report(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples),
                "note": "sampled during warm-up and the timed region"}


# ----------------------------------------------------------------- helpers
# Spec figures, reported beside the measured-peak fractions: dense bf16 tensor
# throughput of one B200 and its HBM3e bandwidth (~8 TB/s).
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0


def tensor_peak(clocks, peak_burst, peak_sust, peak_kind):
    """The bf16 denominator that matches the clocks the kernel ran at: the
    sustained GEMM figure (measured back to back under the power cap) only
    when the sampled SM clock sat well below its maximum with the power cap
    active, else the burst figure."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = ("sw_power_cap" in clocks.get("reasons", []) and mhz is not None and mx
              and mhz < 0.9 * mx)
    if capped:
        return peak_sust, "%s bf16 sustained (SM clock %d of %d MHz, power cap)" % (
            peak_kind, mhz, mx), {"frac_of_burst_peak_at": peak_burst}
    return peak_burst, "%s bf16 burst" % peak_kind, {"frac_of_sustained_peak_at": peak_sust}


def roofline_tensor(achieved, clocks, peaks, **extra):
    _, peak_burst, peak_sust, peak_kind = peaks
    peak, kind, other = tensor_peak(clocks, peak_burst, peak_sust, peak_kind)
    alt_name, alt_peak = next(iter(other.items()))
    line = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_kind": kind,
            alt_name.replace("_at", ""): round(achieved / alt_peak, 4),
            "frac_of_nominal": round(achieved / NOMINAL_BF16_TFLOPS, 4)}
    line.update(extra)
    return line


def roofline_hbm(achieved, hbm, peak_kind, **extra):
    line = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_kind": "%s HBM copy" % peak_kind,
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4)}
    line.update(extra)
    return line


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


HOST_MARK = "// ----------------------------------------------------------------- host ---"


def _code_tokens(text):
    """Source text without // and /* */ comments, whitespace collapsed: what
    the compiler sees, so that editing a comment keeps the hash."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def prefill_device_sha():
    """Hash of the prefill kernels' device code: fa_prefill.cu up to its host
    section, plus the shared device helpers (fa_common.cuh), comments and
    whitespace left out.  A DRAM traffic record taken with ncu is only
    reported while this hash is unchanged."""
    h = hashlib.sha256()
    src = open(os.path.join(CSRC, "fa_prefill.cu")).read()
    cut = src.find(HOST_MARK)
    h.update(_code_tokens(src[:cut] if cut >= 0 else src).encode())
    h.update(_code_tokens(open(os.path.join(CSRC, "fa_common.cuh")).read()).encode())
    return h.hexdigest()[:16]


def kernel_traffic(workload):
    """DRAM bytes per FULL prefill launch of `workload` from the committed ncu
    record (profiles/), if it was taken on the current device code and on
    this workload; else None.  Returns (bytes, record's workload, reason)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None, "no ncu record"
    kv = {}
    for line in open(TRAFFIC_FILE):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("device_code_sha256_16") != prefill_device_sha():
        return None, kv.get("workload"), "ncu record is of other device code"
    if kv.get("workload", "").split(" ")[0] != workload:
        return None, kv.get("workload"), "ncu record is of another workload"
    try:
        return float(kv["dram_bytes_per_full_launch"]), kv.get("workload"), "ncu, same code"
    except (KeyError, ValueError):
        return None, kv.get("workload"), "ncu record unreadable"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# -------------------------------------------------------------- our arm
def stack_plan(wl):
    """(number of layers, set of SPARSE layers, decode token per layer?,
    rotated input sets) of one step of a prefill workload."""
    if wl.layers > 1:     # routed stack: a seeded half of the layers biased to SPARSE
        rng = np.random.default_rng(wl.seed)
        sparse = set(rng.choice(wl.layers, size=wl.layers // 2, replace=False).tolist())
        return wl.layers, sparse, False, 1
    if wl.S >= 65536:     # one layer per mode at long context (5 GiB per layer > L2)
        return 2, {1}, True, 1
    return 2, {1}, True, N_INPUT_SETS


class Step:
    """Device buffers of one input set and the launches of one step."""

    def __init__(self, wl, seed, dev, capi, inputs, n_layers=2, sparse_layers=(1,),
                 with_decode=True):
        self.wl, self.dev, self.with_decode = wl, dev, with_decode
        B, S, Hq, Hkv = wl.B, wl.S, wl.Hq, wl.Hkv
        self.layers = []
        for li in range(n_layers):
            bias = (0.0, 0.1) if li in sparse_layers else (0.1, 0.0)
            q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed + 7919 * li, device=dev)
            w1, b1, w2, b2 = inputs.router_weights(Hq * 128, wl.hidden, seed, li, b2=bias)
            lay = dict(q=q, k=k, v=v, w1=w1.to(dev), b1=b1.to(dev), w2=w2.to(dev), b2=b2.to(dev),
                       o=torch.empty_like(q), logits=torch.empty(B, 2, device=dev),
                       mode=torch.empty(B, dtype=torch.int32, device=dev), sparse=li in sparse_layers)
            if with_decode:
                lay["qd"] = inputs.randn_bf16((B, Hq, 128), seed + 31 * li + 5, device=dev)
                lay["od"] = torch.empty_like(lay["qd"])
            self.layers.append(lay)
        self.c = capi.cfg(64, wl.sink, wl.window)
        rows, nnz = capi.blocksparse_index_size(S, self.c)
        self.row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=dev)
        self.col_idx = torch.empty(max(1, nnz), dtype=torch.int32, device=dev)
        self.ws = torch.empty(capi.hybrid_workspace_size(B, Hq, 128, wl.hidden),
                              dtype=torch.uint8, device=dev)
        self.dws = torch.empty(capi.decode_workspace_size(B, Hq, Hkv, S), dtype=torch.uint8,
                               device=dev)
        self.seqlens = torch.full((B,), S, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.capi = capi

    def run(self, ev=None):
        """Enqueue one step.  ev: optional {layer: (start, end)} events
        recorded around that layer's routed attention call."""
        capi, c = self.capi, self.c
        L = capi.lib()
        rc = L.fa_blocksparse_index(self.wl.S, c, capi._ptr(self.row_ptr),
                                    capi._ptr(self.col_idx), capi._stream(self.dev))
        capi._check("fa_blocksparse_index", rc)
        for li, lay in enumerate(self.layers):
            e = ev.get(li) if ev else None
            if e is not None:
                e[0].record()
            capi.hybrid_layer(lay["q"], lay["k"], lay["v"], lay["w1"], lay["b1"], lay["w2"],
                              lay["b2"], self.row_ptr, self.col_idx, c, o=lay["o"],
                              logits=lay["logits"], mode=lay["mode"], workspace=self.ws,
                              status=self.status)
            if e is not None:
                e[1].record()
            if self.with_decode:
                capi.attn_decode(lay["qd"], lay["k"], lay["v"], self.seqlens,
                                 mode_dev=lay["mode"], c=c, o=lay["od"], workspace=self.dws,
                                 status=self.status)


def time_kernel_alone(fn, reps=5):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fn()
    torch.cuda.synchronize()
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / reps


def cpu_inputs(wl, qkv_bits=None):
    """Host data of the oracle's sample: the bf16 bits of Q/K/V (given, or
    drawn on the CPU with the workload's seeds) and the dense block mask."""
    import oracle
    from block_sparse_attention_layerrouter_b200 import inputs
    if qkv_bits is None:
        q, k, v = inputs.qkv(wl.B, wl.S, wl.Hq, wl.Hkv, 128, wl.seed, device="cpu")
        qkv_bits = (inputs.bits(q), inputs.bits(k), inputs.bits(v))
        del q, k, v
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(wl.S, 64, wl.sink, wl.window))
    return qkv_bits + (mask,)


def cpu_baseline(wl, budget_s=15.0, data=None, seed=None):
    """The oracle as it stands, on the host cores, on a bounded sample of the
    workload: seeded query rows, each computed once as a row of the FULL
    layer and once as a row of the SPARSE layer; scaled to TFLOP/s by the
    algorithmic FLOPs of the rows computed (4*D*(attended pairs))."""
    import oracle
    qb, kb, vb, mask = data if data is not None else cpu_inputs(wl)
    S, Hq = wl.S, wl.Hq
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    flops, elapsed, nrows = 0.0, 0.0, 0
    chunk = 64 if S <= 32768 else 16
    oracle.attention_rows(qb, kb, vb, 0.1, np.array([[0, 0, 0]]))   # load + warm
    while elapsed < budget_s:
        ts = rng.integers(0, S, size=chunk)
        hs = rng.integers(0, Hq, size=chunk)
        rows = np.stack([np.zeros(chunk, np.int64), hs, ts], axis=1)
        t0 = time.perf_counter()
        oracle.attention_rows(qb, kb, vb, 1 / math.sqrt(128), rows)           # full layer rows
        oracle.attention_rows(qb, kb, vb, 1 / math.sqrt(128), rows, mask)     # sparse layer rows
        elapsed += time.perf_counter() - t0
        full_pairs = float(np.sum(ts + 1))
        sparse_pairs = 0.0
        for t in ts:
            blocks = np.nonzero(mask[t // 64])[0]
            sparse_pairs += float(np.sum(np.minimum(blocks * 64 + 64, t + 1) - blocks * 64))
        flops += 4.0 * 128 * (full_pairs + sparse_pairs)
        nrows += 2 * chunk
    return {"value": flops / elapsed / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d query rows (random head and position; each row once in the full and "
                      "once in the sparse layer) of %s, %.1f s of oracle time; TFLOP/s from the "
                      "rows' attended pairs" % (nrows, wl.name, elapsed)}


def setup_device(args):
    from block_sparse_attention_layerrouter_b200 import build, capi
    ws, rank, local = dist_env()
    if ws > 1 and not torch.distributed.is_initialized():
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        build.build()
    if ws > 1:
        torch.distributed.barrier()
    capi.lib()
    return ws, rank, dev


def sync_all(ws):
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(ms, ws, dev):
    if ws > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return ms


def base_line(args, wl, ws, ms, unit, value):
    return {"metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 Q/K/V; router weights N(0,0.02)); stands in "
                    "for LongBench-E/RULER prompts of this shape"}


def prefill_config(wl, ws):
    """The `config` of a prefill workload's line; both arms print this dict."""
    n_layers, sparse_layers, with_decode, n_sets = stack_plan(wl)
    layer_bytes = wl.B * wl.S * 128 * 2 * (2 * wl.Hq + 2 * wl.Hkv)    # Q, O, K, V
    return {
        "workload": wl.name, "B": wl.B, "S": wl.S, "Hq": wl.Hq, "Hkv": wl.Hkv, "D": 128,
        "block": 64, "sink": wl.sink, "window": wl.window,
        "router": "%d->%d->2" % (wl.Hq * 128, wl.hidden),
        "step": "index + %d routed layers (%d FULL, %d SPARSE)%s" % (
            n_layers, n_layers - len(sparse_layers), len(sparse_layers),
            " + 1 decode token each" if with_decode else ""),
        "parallelism": "replicas (dp%d, no collective)" % ws if ws > 1 else "single GPU",
        "l2": "inputs %s than L2 (126 MB): %d input set(s) of %.2f GB, rotated" % (
            "larger" if n_layers * layer_bytes > 126e6 else "SMALLER", n_sets,
            n_layers * layer_bytes / 1e9)}


def run_ours(args, wl):
    from block_sparse_attention_layerrouter_b200 import capi, inputs
    ws, rank, dev = setup_device(args)
    headline = wl.name == DEFAULT_WORKLOAD and not args.no_sections
    sections = {}
    if headline:     # the 8K layer first, on a GPU not yet heated by the long launches
        sections[LAYER8K_WORKLOAD] = layer_kernels_section(WORKLOADS_()[LAYER8K_WORKLOAD], dev)
        torch.cuda.empty_cache()
    n_layers, sparse_layers, with_decode, n_sets = stack_plan(wl)
    sets = [Step(wl, wl.seed + 101 * i, dev, capi, inputs, n_layers, sparse_layers, with_decode)
            for i in range(n_sets)]
    full_layer = min(li for li in range(n_layers) if li not in sparse_layers)
    sparse_layer = min(sparse_layers)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev)
    sampler.start()
    for i in range(args.warmup):
        sets[i % n_sets].run()
    sync_all(ws)
    ev = [{li: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for li in (full_layer, sparse_layer)} for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_launch0 = capi.kernel_launches()
    t0.record()
    for i in range(args.steps):
        sets[i % n_sets].run(ev[i])
    t1.record()
    n_launch = capi.kernel_launches() - n_launch0   # kernels enqueued in the timed loop
    sync_all(ws)
    sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), ws, dev)
    ms_full = [e[full_layer][0].elapsed_time(e[full_layer][1]) for e in ev]
    ms_sparse = [e[sparse_layer][0].elapsed_time(e[sparse_layer][1]) for e in ev]
    status = max(int(s.status.item()) for s in sets)
    modes = [int(l["mode"][0].item()) for l in sets[0].layers]
    want = [1 if li in sparse_layers else 0 for li in range(n_layers)]
    assert status == 0, "device status %d" % status

    # ---- the layer kernels each timed alone (breakdown only, not the headline)
    s0 = sets[0]
    lay_f, lay_s = s0.layers[full_layer], s0.layers[sparse_layer]
    reps = 3 if wl.S >= 65536 else 10
    comp = {}
    comp["prefill_full_ms"] = time_kernel_alone(
        lambda: capi.attn_prefill_full(lay_f["q"], lay_f["k"], lay_f["v"], o=lay_f["o"]), reps)
    comp["prefill_sparse_ms"] = time_kernel_alone(
        lambda: capi.attn_prefill_blocksparse(lay_s["q"], lay_s["k"], lay_s["v"], s0.row_ptr,
                                              s0.col_idx, o=lay_s["o"]), reps)
    comp["router_ms"] = time_kernel_alone(
        lambda: capi.router_decide(lay_f["q"], lay_f["w1"], lay_f["b1"], lay_f["w2"],
                                   lay_f["b2"], logits=lay_f["logits"], mode=lay_f["mode"],
                                   workspace=s0.ws))
    cpu_data = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        from block_sparse_attention_layerrouter_b200 import inputs as _in
        cpu_data = cpu_inputs(wl, (_in.bits(lay_f["q"]), _in.bits(lay_f["k"]),
                                   _in.bits(lay_f["v"])))
    del sets, s0, lay_f, lay_s
    torch.cuda.empty_cache()

    e2e = run_e2e(args, wl, dev, capi, inputs, ws) if with_decode else None
    torch.cuda.empty_cache()
    if headline:
        sections["decode"] = decode_section(args, WORKLOADS_()[DECODE_WORKLOAD], dev, ws, rank)
        torch.cuda.empty_cache()
    if rank != 0:
        return None
    hbm, peak_burst, peak_sust, peak_kind = measured_peaks()
    f_full = flops_full(wl)
    f_sparse = flops_sparse_exact(wl)
    f_sparse_exec = 4.0 * 128 * wl.Hq * wl.B * csr_nnz(wl.S, wl.sink, wl.window) * 64 * 64
    step_flops = step_flops_of(wl, n_layers, sparse_layers, with_decode)
    value = ws * step_flops / (ms / args.steps * 1e-3) / 1e12
    avg_full_ms, avg_sparse_ms = statistics.mean(ms_full), statistics.mean(ms_sparse)
    achieved = f_full / (avg_full_ms * 1e-3) / 1e12
    traffic, traffic_wl, traffic_note = kernel_traffic(wl.name)
    comp.update({
        "prefill_full_in_step_ms": avg_full_ms,
        "prefill_sparse_in_step_ms": avg_sparse_ms,
        "prefill_full_tflops": f_full / (comp["prefill_full_ms"] * 1e-3) / 1e12,
        "prefill_sparse_exec_tflops": f_sparse_exec / (comp["prefill_sparse_ms"] * 1e-3) / 1e12,
        "prefill_sparse_exec_frac_of_burst": f_sparse_exec / (comp["prefill_sparse_ms"] * 1e-3)
        / 1e12 / peak_burst,
        "prefill_sparse_exec_in_step_tflops": f_sparse_exec / (avg_sparse_ms * 1e-3) / 1e12,
        "prefill_sparse_exact_tflops": f_sparse / (comp["prefill_sparse_ms"] * 1e-3) / 1e12,
        "routed_modes_match_plan": modes == want,
        "device_status": status,
    })
    line = base_line(args, wl, ws, ms, "TFLOP/s", value)
    line["config"] = prefill_config(wl, ws)
    line["clocks"] = sampler.report()
    line["roofline"] = roofline_tensor(
        achieved, line["clocks"], (hbm, peak_burst, peak_sust, peak_kind),
        kernel="prefill2::prefill2_kernel, FULL layer of the step (CUDA events around "
               "fa_hybrid_layer: router kernels included, %.3f ms of it alone)" % comp["router_ms"],
        traffic=traffic, traffic_source=traffic_note, traffic_workload=traffic_wl,
        algorithmic_flops_per_launch=f_full, avg_launch_ms=round(avg_full_ms, 4),
        sparse_layer={"kernel": "prefill2::prefill2_kernel, SPARSE layer of the step",
                      "avg_launch_ms": round(avg_sparse_ms, 4),
                      "executed_flops_per_launch": f_sparse_exec,
                      "achieved_exec_tflops": round(f_sparse_exec / (avg_sparse_ms * 1e-3)
                                                    / 1e12, 2)})
    if wl.S >= 65536 or n_layers > 2:
        nl = 36 if wl.S >= 65536 else n_layers
        tf, tsp = avg_full_ms, avg_sparse_ms
        tfa, tspa = comp["prefill_full_ms"], comp["prefill_sparse_ms"]
        line["hybrid_vs_full"] = {
            "layers": nl, "split": "50/50",
            "t_full_layer_ms": round(tf, 3), "t_sparse_layer_ms": round(tsp, 3),
            "hybrid_ms": round(nl / 2 * (tf + tsp), 2), "all_full_ms": round(nl * tf, 2),
            "speedup": round((nl * tf) / (nl / 2 * (tf + tsp)), 4),
            "speedup_layers_alone": round((nl * tfa) / (nl / 2 * (tfa + tspa)), 4),
            "note": "layer times from the timed steps (routed layers, router included); "
                    "projection = %d/2 FULL + %d/2 SPARSE layers vs %d FULL" % (nl, nl, nl),
            "pages_context": "up to 2.8x prefill at 256K (hardware not stated)"}
    line["e2e"] = e2e
    line["gpu_launches"] = n_launch
    line["components"] = {k: (round(v, 4) if isinstance(v, float) else v) for k, v in comp.items()}
    line.update(sections)
    if cpu_data is not None:
        line["cpu_baseline"] = cpu_baseline(wl, data=cpu_data)
    return line


def WORKLOADS_():
    from block_sparse_attention_layerrouter_b200.inputs import WORKLOADS
    return WORKLOADS


def step_flops_of(wl, n_layers, sparse_layers, with_decode):
    ns = len(sparse_layers)
    nf = n_layers - ns
    f = nf * flops_full(wl) + ns * flops_sparse_exact(wl)
    if with_decode:
        keys = nf * decode_keys(wl.S, 0, wl.sink, wl.window) + \
            ns * decode_keys(wl.S, 1, wl.sink, wl.window)
        f += 4.0 * 128 * wl.Hq * wl.B * keys
    return f


def layer_kernels_section(wl, dev):
    """FULL and SPARSE prefill of one layer of `wl`, each launched alone
    (the 8K-context layer: several full waves of work items per launch)."""
    from block_sparse_attention_layerrouter_b200 import capi, inputs
    q, k, v = inputs.qkv(wl.B, wl.S, wl.Hq, wl.Hkv, 128, wl.seed, device=dev)
    o = torch.empty_like(q)
    c = capi.cfg(64, wl.sink, wl.window)
    rp, ci = capi.blocksparse_index(wl.S, c, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sampler = ClockSampler(dev, period_s=0.005)
    sampler.start()
    tf = time_kernel_alone(lambda: capi.attn_prefill_full(q, k, v, o=o, status=status), 20)
    ts = time_kernel_alone(lambda: capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o,
                                                                 status=status), 20)
    torch.cuda.synchronize()
    sampler.stop()
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    _, peak_burst, peak_sust, _ = measured_peaks()
    f_full = flops_full(wl)
    f_exec = 4.0 * 128 * wl.Hq * wl.B * csr_nnz(wl.S, wl.sink, wl.window) * 64 * 64
    return {"config": {"B": wl.B, "S": wl.S, "Hq": wl.Hq, "Hkv": wl.Hkv, "window": wl.window,
                       "sink": wl.sink},
            "timing": "each kernel alone, 20 launches on one input set (0.34 GB), CUDA events, "
                      "before the long launches of the run",
            "clocks": sampler.report(),
            "prefill_full_ms": round(tf, 4),
            "prefill_full_tflops": round(f_full / (tf * 1e-3) / 1e12, 2),
            "prefill_full_frac_of_burst": round(f_full / (tf * 1e-3) / 1e12 / peak_burst, 4),
            "prefill_sparse_ms": round(ts, 4),
            "prefill_sparse_exec_tflops": round(f_exec / (ts * 1e-3) / 1e12, 2),
            "prefill_sparse_exec_frac_of_burst": round(f_exec / (ts * 1e-3) / 1e12 / peak_burst,
                                                       4),
            "prefill_sparse_exact_tflops": round(flops_sparse_exact(wl) / (ts * 1e-3) / 1e12, 2)}


def run_e2e(args, wl, dev, capi, inputs, ws):
    """Same step through the public API with host buffers: per step, copy
    the layers' Q/K/V and decode queries from pinned host memory, run, and
    read the layers' outputs back.  The copies are pipelined across steps:
    two device buffer sets, the inputs of step i+1 going up on one copy
    stream and the outputs of step i-1 coming down on another while step i
    computes (PCIe is full duplex)."""
    n_layers, sparse_layers, with_decode, _ = stack_plan(wl)
    steps = [Step(wl, wl.seed, dev, capi, inputs, n_layers, sparse_layers, with_decode)
             for _ in range(2)]
    host = []
    for lay in steps[0].layers:
        host.append([lay[n].cpu().pin_memory() for n in ("q", "k", "v", "qd")])
    # One host output set: the D2H copies run in order on one stream.
    outs = [(torch.empty(lay["o"].shape, dtype=lay["o"].dtype).pin_memory(),
             torch.empty(lay["od"].shape, dtype=lay["od"].dtype).pin_memory())
            for lay in steps[0].layers]
    h2d = sum(t.numel() * t.element_size() for hs in host for t in hs)
    d2h = sum(t.numel() * t.element_size() for o in outs for t in o)
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_comp = torch.cuda.current_stream(dev)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("up", "comp", "down")}
    started = [False, False]

    def one(i):
        b = i % 2
        st = steps[b]
        with torch.cuda.stream(s_up):
            if started[b]:
                s_up.wait_event(ev["comp"][b])          # step i-2 is done reading its inputs
            for li, lay in enumerate(st.layers):
                for name, t in zip(("q", "k", "v", "qd"), host[li]):
                    lay[name].copy_(t, non_blocking=True)
            ev["up"][b].record(s_up)
        s_comp.wait_event(ev["up"][b])
        if started[b]:
            s_comp.wait_event(ev["down"][b])            # step i-2's outputs have left
        st.run()
        ev["comp"][b].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev["comp"][b])
            for li, lay in enumerate(st.layers):
                outs[li][0].copy_(lay["o"], non_blocking=True)
                outs[li][1].copy_(lay["od"], non_blocking=True)
            ev["down"][b].record(s_down)
        started[b] = True

    for i in range(max(1, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    sync_all(ws)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(s_comp)
    s_up.wait_event(s)
    for i in range(args.steps):
        one(args.warmup + i)
    s_comp.wait_event(ev["down"][(args.warmup + args.steps - 1) % 2])
    s_comp.wait_event(ev["down"][(args.warmup + args.steps - 2) % 2])
    e.record(s_comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), ws, dev)
    flops = step_flops_of(wl, n_layers, sparse_layers, with_decode)
    return {"value": round(ws * flops / (ms / args.steps * 1e-3) / 1e12, 3),
            "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / args.steps, 4),
            "note": "copies pipelined across steps (two device buffer sets, separate H2D "
                    "and D2H streams)"}


# ------------------------------------------------------------ decode stack
DECODE_CACHE_SETS = 8


def decode_measure(wl, dev, ws, steps, warmup, min_seconds=0.0):
    """Decode step of a 32-layer model: one token per sequence per layer,
    layers alternating FULL / SPARSE (16 + 16, fixed by the router at
    prefill).  Each layer reads its own KV cache; 8 distinct cache sets (4 GiB
    each) are rotated over the 32 layers, so consecutive reads of one set are
    8 layers (>= 16 GiB of other traffic) apart and come from HBM.  With
    min_seconds > 0 the timed step count is raised until the timed region
    lasts at least that long (estimated from the warm-up steps).  Returns a
    dict of measurements (every rank) or raises on a device error."""
    from block_sparse_attention_layerrouter_b200 import capi, inputs
    B, L, Hq, Hkv = wl.B, wl.decode_len, wl.Hq, wl.Hkv
    caches = []
    max_pages = L // 64
    bt = inputs.page_table(B, max_pages, wl.seed).to(dev) if wl.paged else None
    ksc = inputs.fp8_scales(Hkv, wl.seed).to(dev) if wl.kv_fp8 else None
    vsc = inputs.fp8_scales(Hkv, wl.seed + 1).to(dev) if wl.kv_fp8 else None
    kv_dtype = capi.FA_KV_FP8_E4M3 if wl.kv_fp8 else capi.FA_KV_BF16
    for i in range(DECODE_CACHE_SETS):
        if wl.kv_fp8:
            shape = (B * max_pages, 64, Hkv, 128)
            caches.append((inputs.fp8_codes(shape, wl.seed + 17 * i, device=dev),
                           inputs.fp8_codes(shape, wl.seed + 17 * i + 5, device=dev)))
            continue
        _, kc, vc = inputs.decode_inputs(B, L, Hq, Hkv, 128, wl.seed + 17 * i, device=dev)
        if wl.paged:
            kc = kc.view(B * max_pages, 64, Hkv, 128)
            vc = vc.view(B * max_pages, 64, Hkv, 128)
        caches.append((kc, vc))
    qs = [inputs.randn_bf16((B, Hq, 128), wl.seed + 1000 + li, device=dev)
          for li in range(wl.layers)]
    outs = [torch.empty_like(q) for q in qs]
    sl = torch.full((B,), L, dtype=torch.int32, device=dev)
    c = capi.cfg(64, wl.sink, wl.window)
    wsb = torch.empty(capi.decode_workspace_size(B, Hq, Hkv, L), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    modes = [li % 2 for li in range(wl.layers)]      # 0 FULL, 1 SPARSE

    def step(ev=None):
        for li in range(wl.layers):
            kc, vc = caches[li % DECODE_CACHE_SETS]
            if ev is not None and li == 0:
                ev[0].record()
            if wl.paged:
                capi.attn_decode_paged(qs[li], kc, vc, bt, sl, kv_dtype, ksc, vsc, modes[li], c,
                                       o=outs[li], workspace=wsb, status=status)
            else:
                capi.attn_decode(qs[li], kc, vc, sl, modes[li], c, o=outs[li], workspace=wsb,
                                 status=status)
            if ev is not None and li == 0:
                ev[1].record()

    sampler = ClockSampler(dev)
    sampler.start()
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step()
    w0.record()
    for _ in range(max(1, warmup - 1)):
        step()
    w1.record()
    sync_all(ws)
    if min_seconds > 0:
        est = w0.elapsed_time(w1) / max(1, warmup - 1)
        est = max_over_ranks(est, ws, dev)       # every rank times the same count
        steps = max(steps, int(math.ceil(min_seconds * 1e3 / max(est, 1e-3))))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_launch0 = capi.kernel_launches()
    t0.record()
    for i in range(steps):
        step(evs[i])
    t1.record()
    n_launch = capi.kernel_launches() - n_launch0   # kernels enqueued in the timed loop
    sync_all(ws)
    sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), ws, dev)
    full_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    if wl.paged:
        sparse_ms = time_kernel_alone(lambda: capi.attn_decode_paged(
            qs[1], *caches[1], bt, sl, kv_dtype, ksc, vsc, 1, c, o=outs[1], workspace=wsb))
        # KV append of one token for all sequences, alone (positions L-9 ..).
        sl_app = torch.full((B,), L - 9, dtype=torch.int32, device=dev)
        kn = inputs.randn_bf16((B, Hkv, 128), wl.seed + 2, device=dev)
        append_ms = time_kernel_alone(lambda: capi.kv_append_paged(
            kn, kn, caches[0][0], caches[0][1], bt, sl_app, kv_dtype, ksc, vsc), reps=5)
    else:
        sparse_ms = time_kernel_alone(lambda: capi.attn_decode(qs[1], *caches[1], sl, 1, c,
                                                               o=outs[1], workspace=wsb))
        append_ms = None
    # FULL layer alone on one cache (a burst, 10 launches): the kernel's own rate.
    full_alone_ms = time_kernel_alone(lambda: capi.attn_decode(
        qs[0], *caches[0], sl, 0, c, o=outs[0], workspace=wsb), reps=10) if not wl.paged else None
    # e2e: the caches are device-resident state; per step the 32 layers'
    # query tokens go up from pinned host memory and their outputs come back.
    hq = [q.cpu().pin_memory() for q in qs]
    ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]

    def step_e2e():
        for li in range(wl.layers):
            qs[li].copy_(hq[li], non_blocking=True)
        step()
        for li in range(wl.layers):
            ho[li].copy_(outs[li], non_blocking=True)

    for _ in range(2):
        step_e2e()
    sync_all(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step_e2e()
    e1.record()
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), ws, dev)
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    hbm, _, _, peak_kind = measured_peaks()
    kv_row = 2 * Hkv * 128 * (1 if wl.kv_fp8 else 2)         # K and V bytes per token
    qo = 2 * B * Hq * 128 * 2
    full_bytes = B * kv_row * decode_keys(L, 0, wl.sink, wl.window) + qo
    sparse_bytes = B * kv_row * decode_keys(L, 1, wl.sink, wl.window) + qo
    step_bytes = sum(full_bytes if m == 0 else sparse_bytes for m in modes)
    clocks = sampler.report()
    out = {
        "value": round(ws * step_bytes / (ms / steps * 1e-3) / 1e9, 1), "unit": "GB/s",
        "steps": steps, "ms_per_step": round(ms / steps, 4), "timed_s": round(ms / 1e3, 3),
        "config": {"workload": wl.name, "B": B, "L": L, "Hq": Hq, "Hkv": Hkv, "D": 128,
                   "layers": wl.layers, "split": "16 FULL + 16 SPARSE (alternating)",
                   "sink": wl.sink, "window": wl.window,
                   "cache": ("paged (64-token pages, seeded random order), " if wl.paged
                             else "contiguous, ") + ("E4M3 + per-head scales" if wl.kv_fp8
                                                     else "bf16"),
                   "l2": "inputs larger than L2: %d cache sets of %.2f GB rotated" % (
                       DECODE_CACHE_SETS,
                       2 * caches[0][0].numel() * caches[0][0].element_size() / 1e9)},
        "clocks": clocks,
        "roofline": roofline_hbm(
            full_bytes / (full_ms * 1e-3) / 1e9, hbm, peak_kind,
            kernel="decode::decode_kernel + combine_kernel (FULL layer of the step)",
            traffic=None, algorithmic_bytes_per_launch=full_bytes,
            avg_launch_ms=round(full_ms, 4)),
        "e2e": {"value": round(ws * step_bytes / (ms_e2e / steps * 1e-3) / 1e9, 1),
                "unit": "GB/s", "h2d_bytes_per_step": sum(t.numel() * 2 for t in hq),
                "d2h_bytes_per_step": sum(t.numel() * 2 for t in ho),
                "note": "KV caches are device-resident decode state"},
        "gpu_launches": n_launch,
        "components": {
            "decode_full_layer_ms": round(full_ms, 4),
            "decode_sparse_layer_ms": round(sparse_ms, 4),
            "decode_sparse_gbs": round(sparse_bytes / (sparse_ms * 1e-3) / 1e9, 1),
            "all_full_step_ms_est": round(wl.layers * full_ms, 3),
            "hybrid_vs_all_full": round(wl.layers * full_ms / (ms / steps), 3),
            "pages_context": "up to 2.0x decode at 256K (hardware not stated)"}}
    if full_alone_ms is not None:
        out["components"]["decode_full_layer_alone_ms"] = round(full_alone_ms, 4)
        out["components"]["decode_full_layer_alone_gbs"] = round(
            full_bytes / (full_alone_ms * 1e-3) / 1e9, 1)
        out["components"]["decode_full_layer_alone_frac_of_hbm"] = round(
            full_bytes / (full_alone_ms * 1e-3) / 1e9 / hbm, 4)
    if append_ms is not None:
        out["components"]["kv_append_ms"] = round(append_ms, 4)
    del caches
    return out


def decode_section(args, wl, dev, ws, rank):
    """The 32-layer decode step inside the headline line, timed for at least
    one second whatever --steps is, so the clock record covers it."""
    d = decode_measure(wl, dev, ws, args.steps, args.warmup, min_seconds=1.0)
    return d if rank == 0 else None


def run_decode(args, wl):
    ws, rank, dev = setup_device(args)
    d = decode_measure(wl, dev, ws, args.steps, args.warmup)
    if rank != 0:
        return None
    line = base_line(args, wl, ws, d["ms_per_step"] * args.steps, "GB/s", d["value"])
    for k in ("config", "clocks", "roofline", "e2e", "gpu_launches", "components"):
        line[k] = d[k]
    return line


# ------------------------------------------------ variable-length serving
def run_varlen(args, wl):
    """One routed layer over a packed batch of requests of different lengths:
    CSR + fa_hybrid_layer_varlen (router per request on the device, then one
    persistent attention launch over every request in its own mode)."""
    import oracle  # pair counting only (host arithmetic of the pattern)
    from block_sparse_attention_layerrouter_b200 import capi, inputs
    ws, rank, dev = setup_device(args)
    lengths = inputs.varlen_lengths(wl.B, wl.S, wl.seed)
    T = int(lengths.sum())
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=dev)
    q = inputs.randn_bf16((T, wl.Hq, 128), wl.seed, device=dev)
    k = inputs.randn_bf16((T, wl.Hkv, 128), wl.seed + 100, device=dev)
    v = inputs.randn_bf16((T, wl.Hkv, 128), wl.seed + 200, device=dev)
    o = torch.empty_like(q)
    w1, b1, w2, b2 = [t.to(dev) for t in inputs.router_weights(wl.Hq * 128, wl.hidden, wl.seed)]
    c = capi.cfg(64, wl.sink, wl.window)
    rows, nnz = capi.blocksparse_index_size(wl.S, c)
    rp = torch.empty(rows + 1, dtype=torch.int32, device=dev)
    ci = torch.empty(nnz, dtype=torch.int32, device=dev)
    logits = torch.empty(wl.B, 2, device=dev)
    mode = torch.empty(wl.B, dtype=torch.int32, device=dev)
    wsb = torch.empty(int(capi.lib().fa_hybrid_varlen_workspace_size(wl.B, T, wl.Hq, 128,
                                                                      wl.hidden)),
                      dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(ev=None):
        capi._check("fa_blocksparse_index", capi.lib().fa_blocksparse_index(
            wl.S, c, capi._ptr(rp), capi._ptr(ci), capi._stream(dev)))
        if ev is not None:
            ev[0].record()
        capi.hybrid_layer_varlen(q, k, v, cu, wl.S, w1, b1, w2, b2, rp, ci, c, o=o,
                                 logits=logits, mode=mode, workspace=wsb, status=status)
        if ev is not None:
            ev[1].record()

    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(args.warmup):
        step()
    sync_all(ws)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_launch0 = capi.kernel_launches()
    t0.record()
    for i in range(args.steps):
        step(evs[i])
    t1.record()
    n_launch = capi.kernel_launches() - n_launch0   # kernels enqueued in the timed loop
    sync_all(ws)
    sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), ws, dev)
    layer_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    modes = mode.cpu().tolist()
    # The same packed batch with every request in FULL mode (one varlen launch):
    # what the routing saves on this batch.
    vws = torch.empty(int(capi.lib().fa_varlen_workspace_size(wl.B, T)), dtype=torch.uint8,
                      device=dev)
    full_ms = time_kernel_alone(lambda: capi.attn_prefill_varlen(
        q, k, v, cu, wl.S, mode=0, o=o, workspace=vws, status=status))
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    if rank != 0:
        return None
    flops = 0.0
    for L, m in zip(lengths.tolist(), modes):
        pairs = L * (L + 1) / 2 if m == 0 else oracle.attended_pairs_sparse(L, 64, wl.sink,
                                                                          wl.window)
        flops += 4.0 * 128 * wl.Hq * pairs
    _, peak_burst, peak_sust, peak_kind = measured_peaks()
    value = ws * flops / (ms / args.steps * 1e-3) / 1e12
    achieved = flops / (layer_ms * 1e-3) / 1e12
    line = base_line(args, wl, ws, ms, "TFLOP/s", value)
    line["config"] = {"workload": wl.name, "requests": wl.B, "lengths": lengths.tolist(),
                      "total_tokens": T, "Hq": wl.Hq, "Hkv": wl.Hkv, "D": 128, "sink": wl.sink,
                      "window": wl.window, "routed_modes": modes,
                      "step": "CSR + router per request + one packed attention launch",
                      "l2": "inputs larger than L2 (%.2f GB)" % (
                          (q.numel() * 2 * 2 + k.numel() * 2 * 2) / 1e9)}
    line["clocks"] = sampler.report()
    line["roofline"] = roofline_tensor(
        achieved, line["clocks"], (None, peak_burst, peak_sust, peak_kind),
        kernel="router + varlen prefill2_kernel", traffic=None,
        algorithmic_flops_per_launch=flops, avg_launch_ms=round(layer_ms, 4))
    line["all_full_ms"] = round(full_ms, 4)
    line["routed_speedup_vs_all_full"] = round(full_ms / (ms / args.steps), 3)
    line["e2e"] = None
    line["gpu_launches"] = n_launch
    return line


# ------------------------------------------------------ training step
def run_train(args, wl):
    """One training step of a soft-routed layer: router logits and the soft
    weight r, FULL and SPARSE attention with their LSE (forward), then
    fa_soft_routed_layer_backward for an upstream gradient of the mixed
    output (router weights, Q, K, V through both paths)."""
    from block_sparse_attention_layerrouter_b200 import capi, inputs
    ws, rank, dev = setup_device(args)
    B, S, Hq, Hkv = wl.B, wl.S, wl.Hq, wl.Hkv
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, wl.seed, device=dev)
    dy = inputs.randn_bf16((B, S, Hq, 128), wl.seed + 400, device=dev)
    w1, b1, w2, b2 = [t.to(dev) for t in inputs.router_weights(Hq * 128, wl.hidden, wl.seed)]
    g = inputs.gumbel(B, wl.seed).to(dev)
    c = capi.cfg(64, wl.sink, wl.window)
    rp, ci = capi.blocksparse_index(S, c, device=dev)
    o_f, o_s, y = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    lse_f = torch.empty(B, Hq, S, device=dev)
    lse_s = torch.empty(B, Hq, S, device=dev)
    logits = torch.empty(B, 2, device=dev)
    r = torch.empty(B, device=dev)
    mode = torch.empty(B, dtype=torch.int32, device=dev)
    rws = torch.empty(capi.router_workspace_size(B, Hq, 128, wl.hidden), dtype=torch.uint8,
                      device=dev)
    bws = torch.empty(int(capi.lib().fa_soft_routed_backward_workspace_size(B, S, Hq, Hkv, 128,
                                                                             wl.hidden)),
                      dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        capi.router_decide(q, w1, b1, w2, b2, logits=logits, mode=mode, workspace=rws)
        capi.router_soft(logits, g, tau=1.0, r=r)
        capi.attn_prefill_full(q, k, v, o=o_f, lse=lse_f, status=status)
        capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o_s, lse=lse_s, status=status)
        capi.soft_mix(o_f, o_s, r, y=y)
        return capi.soft_routed_layer_backward(q, k, v, o_f, lse_f, o_s, lse_s, dy, w1, b1, w2, b2,
                                               rp, ci, gumbel=g, tau=1.0, workspace=bws,
                                               status=status)

    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(args.warmup):
        step()
    sync_all(ws)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_launch0 = capi.kernel_launches()
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    n_launch = capi.kernel_launches() - n_launch0   # kernels enqueued in the timed loop
    sync_all(ws)
    sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), ws, dev)
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    if rank != 0:
        return None
    f_full = flops_full(wl)
    f_sparse = 4.0 * 128 * Hq * B * csr_nnz(S, wl.sink, wl.window) * 4096
    flops = 3.5 * (f_full + f_sparse)      # forward 1x, backward 2.5x of each path
    bwd_full_ms = time_kernel_alone(lambda: capi.attn_prefill_backward(
        q, k, v, o_f, lse_f, dy, mode=0))
    _, peak_burst, peak_sust, peak_kind = measured_peaks()
    value = ws * flops / (ms / args.steps * 1e-3) / 1e12
    bwd_achieved = 2.5 * f_full / (bwd_full_ms * 1e-3) / 1e12
    line = base_line(args, wl, ws, ms, "TFLOP/s", value)
    line["config"] = {"workload": wl.name, "B": B, "S": S, "Hq": Hq, "Hkv": Hkv, "D": 128,
                      "sink": wl.sink, "window": wl.window, "hidden": wl.hidden,
                      "step": "router + r + FULL and SPARSE forward with LSE + y = r O_FA + "
                              "(1-r) O_SA + soft-routed backward (router grads, dQ/dK/dV "
                              "through both paths)",
                      "flops": "forward 4*D*Hq*pairs per path (SPARSE: executed 64x64 "
                               "blocks), backward 2.5x the forward",
                      "l2": "Q/K/V/O/dy/accumulators 0.6 GB per step > L2"}
    line["clocks"] = sampler.report()
    line["roofline"] = roofline_tensor(
        bwd_achieved, line["clocks"], (None, peak_burst, peak_sust, peak_kind),
        kernel="backward::bwd_kernel (FULL, alone)", traffic=None,
        algorithmic_flops_per_launch=2.5 * f_full, avg_launch_ms=round(bwd_full_ms, 4))
    line["e2e"] = None
    line["gpu_launches"] = n_launch
    return line


# ------------------------------------------------------- one kernel alone
def run_only(args, wl):
    """Runs a single kernel of the path `warmup + steps` times on the
    workload's shapes (used for ncu captures and quick timing)."""
    from block_sparse_attention_layerrouter_b200 import capi, inputs
    ws, rank, dev = setup_device(args)
    B, Hq, Hkv = wl.B, wl.Hq, wl.Hkv
    S = wl.decode_len or wl.S
    c = capi.cfg(64, wl.sink, wl.window)
    if args.only.startswith("decode_fp8"):
        max_pages = S // 64
        q = inputs.randn_bf16((B, Hq, 128), wl.seed, device=dev)
        kc = inputs.fp8_codes((B * max_pages, 64, Hkv, 128), wl.seed + 100, device=dev)
        vc = inputs.fp8_codes((B * max_pages, 64, Hkv, 128), wl.seed + 200, device=dev)
        bt = inputs.page_table(B, max_pages, wl.seed).to(dev)
        ksc, vsc = inputs.fp8_scales(Hkv, wl.seed).to(dev), inputs.fp8_scales(Hkv, 1).to(dev)
        sl = torch.full((B,), S, dtype=torch.int32, device=dev)
        wsb = torch.empty(capi.decode_workspace_size(B, Hq, Hkv, S), dtype=torch.uint8,
                          device=dev)
        md = 0 if args.only == "decode_fp8_full" else 1
        o = torch.empty_like(q)
        fn = lambda: capi.attn_decode_paged(  # noqa: E731
            q, kc, vc, bt, sl, capi.FA_KV_FP8_E4M3, ksc, vsc, md, c, o=o, workspace=wsb)
        work = B * 2 * Hkv * 128 * 1 * decode_keys(S, md, wl.sink, wl.window) / 1e9
        unit = "GB/s"
    elif args.only.startswith("decode"):
        q, kc, vc = inputs.decode_inputs(B, S, Hq, Hkv, 128, wl.seed, device=dev)
        sl = torch.full((B,), S, dtype=torch.int32, device=dev)
        wsb = torch.empty(capi.decode_workspace_size(B, Hq, Hkv, S), dtype=torch.uint8,
                          device=dev)
        md = 0 if args.only == "decode_full" else 1
        o = torch.empty_like(q)
        fn = lambda: capi.attn_decode(q, kc, vc, sl, md, c, o=o, workspace=wsb)  # noqa: E731
        work = B * 2 * Hkv * 128 * 2 * decode_keys(S, md, wl.sink, wl.window) / 1e9
        unit = "GB/s"
    else:
        q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, wl.seed, device=dev)
        o = torch.empty_like(q)
        rp, ci = capi.blocksparse_index(S, c, device=dev)
        w1, b1, w2, b2 = [t.to(dev) for t in inputs.router_weights(Hq * 128, wl.hidden, wl.seed)]
        unit = "TFLOP/s"
        if args.only == "prefill_full":
            fn = lambda: capi.attn_prefill_full(q, k, v, o=o)  # noqa: E731
            work = flops_full(wl) / 1e12
        elif args.only == "prefill_sparse":
            fn = lambda: capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o)  # noqa: E731
            work = 4.0 * 128 * Hq * B * csr_nnz(S, wl.sink, wl.window) * 4096 / 1e12
        elif args.only in ("backward_full", "backward_sparse"):
            sparse = args.only == "backward_sparse"
            lse = torch.empty(B, Hq, S, device=dev)
            if sparse:
                capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o, lse=lse)
            else:
                capi.attn_prefill_full(q, k, v, o=o, lse=lse)
            do = inputs.randn_bf16((B, S, Hq, 128), wl.seed + 400, device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            bws = torch.empty(capi.attn_backward_workspace_size(B, S, Hq, Hkv), dtype=torch.uint8,
                              device=dev)
            fn = lambda: capi.attn_prefill_backward(  # noqa: E731
                q, k, v, o, lse, do, rp, ci, mode=int(sparse), dq=dq, dk=dk, dv=dv, workspace=bws)
            # 2.5x the forward's FLOPs: S, dP, dV, dK and dQ products per pair.
            if sparse:
                work = 10.0 * 128 * Hq * B * csr_nnz(S, wl.sink, wl.window) * 4096 / 1e12
            else:
                work = 2.5 * flops_full(wl) / 1e12
        elif args.only == "router":
            fn = lambda: capi.router_decide(q, w1, b1, w2, b2)  # noqa: E731
            work = (B * 200 * Hq * 128 * 2 + w1.numel() * 4) / 1e9
            unit = "GB/s"
        else:
            raise SystemExit("unknown --only " + args.only)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / args.steps
    return {"only": args.only, "workload": wl.name, "ms": round(ms, 4),
            "value": round(work / (ms * 1e-3), 2), "unit": unit, "steps": args.steps}


# --------------------------------------------------------- reference arm
def run_reference(args, wl):
    """The oracle as it stands on the host cores, same metric, unit and
    config as our arm; each step a bounded sample of the workload (see
    cpu_baseline).  Under torchrun rank 0 alone runs it."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return None
    if wl.decode_len or wl.varlen or wl.train:
        return {"impl": "reference", "unavailable": "the reference arm times the prefill "
                "workloads only (the oracle's attention rows); %s is not one" % wl.name}
    budget = float(os.environ.get("FA_REF_STEP_S", "4"))
    data = cpu_inputs(wl)
    vals, t_total = [], 0.0
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        r = cpu_baseline(wl, budget_s=budget, data=data, seed=wl.seed + i)
        if i >= args.warmup:
            vals.append(r["value"])
            t_total += time.perf_counter() - t0
    value = statistics.mean(vals)
    r["value"] = value
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "impl": "reference",
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t_total / max(1, args.steps), 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": prefill_config(wl, ws),
            "cpu_baseline": r,
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------- host-only dry run
def run_dry(args, wl):
    """The multi-rank host path without a GPU: gloo process group, barrier,
    a timed host loop, maximum over ranks, one line from rank 0."""
    ws, rank, _ = dist_env()
    if ws > 1 and not torch.distributed.is_initialized():
        from datetime import timedelta
        torch.distributed.init_process_group("gloo", timeout=timedelta(seconds=120))
    dev = torch.device("cpu")
    sync_all(ws)
    t0 = time.perf_counter()
    for _ in range(args.warmup + args.steps):
        torch.ones(64).sum()
    ms = max_over_ranks((time.perf_counter() - t0) * 1e3, ws, dev)
    if rank != 0:
        return None
    line = base_line(args, wl, ws, ms, "TFLOP/s", 0.0)
    line.update({"dry_run": True, "config": prefill_config(wl, ws), "e2e": None,
                 "gpu_launches": 0})
    return line


def relaunch(args) -> int:
    """`--gpus N` outside torchrun: start N ranks of this script through
    torch.distributed.run on this node and return their exit status."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node=%d" % args.gpus, "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 200 for the sub-millisecond 8K step, so the "
                         "clock samples cover the timed region; 20 otherwise)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sections", action="store_true",
                    help="headline workload without the decode and 8K sections")
    ap.add_argument("--dry-run", action="store_true",
                    help="host path only (gloo, no GPU): ranks, barrier, max over ranks")
    ap.add_argument("--only", default=None,
                    help="prefill_full | prefill_sparse | decode_full | decode_sparse | "
                         "decode_fp8_full | decode_fp8_sparse | backward_full | "
                         "backward_sparse | router")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch(args))
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE=%d" % (args.gpus, ws))
    from block_sparse_attention_layerrouter_b200.inputs import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.steps is None:
        args.steps = 200 if (args.impl == "ours" and not args.only
                             and wl.name == LAYER8K_WORKLOAD) else 20
    if args.dry_run:
        line = run_dry(args, wl)
    elif args.impl == "reference":
        line = run_reference(args, wl)
    elif args.only:
        line = run_only(args, wl)
    elif wl.decode_len:
        line = run_decode(args, wl)
    elif wl.varlen:
        line = run_varlen(args, wl)
    elif wl.train:
        line = run_train(args, wl)
    else:
        line = run_ours(args, wl)
    if line is not None:
        print(json.dumps(line), flush=True)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
