#!/usr/bin/env python
"""Benchmark of the B200 triangle multiplicative update.

One step = one pass of the whole layer in both directions (outgoing, then
incoming) over one synthetic pair representation: per direction the prologue,
contraction and epilogue kernels, called through the C ABI. The default
workload is the Boltz-2 crop size N = 768 (bf16, c_z = c_h = 128, per-channel
scale on z). The metric is pair-cells/s (one cell through one direction of the
layer is one pair-cell); algorithmic TFLOP/s is reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) every rank runs an independent replica on its
own GPU; value = cells of all ranks / max time. --mode sharded instead splits one
layer over the ranks (pair_representation_b200.sharded; strong scaling).

Secondary figures on rank 0 at N = 1: every workload per direction
("per_config"), one trimul_backward call per direction at N = 768
("backward"; --backward-only times just that), one windowed atom-attention
call on 8 x 18432 atoms ("atom_attention"; --attention-only) and the MXFP8
contraction beside the bf16 one at N = 768, 2048 and 3605 ("mxfp8";
--mxfp8-only).

Timing: CUDA events on the launching stream; L2 is flushed (512 MB write)
before every step and the flush is outside the timed events; a barrier and a
device synchronize bracket the K timed steps on every rank. The step (both
directions, six stage calls) is captured once as a CUDA graph and replayed:
dependent kernels then start under 1 us apart instead of about 2 us. The timed
steps carry events only at step boundaries; the per-kernel breakdown and the
roofline come from a second graph with a timing event before every kernel,
replayed for another K steps; the same step launched eagerly is reported as
`eager_ms_per_step`.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "trimul pair-cells/s and TFLOP/s at N=768 bf16 (% of B200 tensor peak)"
UNIT = "pair-cells/s"
DEFAULT_WORKLOAD = 3
FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (HGX HBM3e bandwidth, dense bf16 tensor rate), reported beside the measured ones.
NOMINAL_PEAKS = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
KERNELS = ("prologue_tc_kernel", "contract_tc_kernel", "epilogue_tc_kernel")


def flops_per_cell(N: int) -> int:
    """Algorithmic FLOP per cell and direction: projections 2*(4*128*128 + 128*128 + 128*128), contraction 2*N*128."""
    return 196608 + 256 * N


def kernel_algorithmic(N: int):
    """Per launch: (quantity, unit, bound) of each kernel's algorithmic work."""
    cells = N * N
    return {
        "prologue_tc_kernel": (cells * (256 + 2 + 512) + 4 * 128 * 128 * 2, "bytes", "hbm"),
        "contract_tc_kernel": (2 * N ** 3 * 128, "flop", "tensor"),
        "epilogue_tc_kernel": (cells * (256 + 256 + 256) + 2 * 128 * 128 * 2, "bytes", "hbm"),
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(kernel: str) -> str:
    files = {"prologue_tc_kernel": ("prologue_tc.cu", "tile_ops.cuh", "mx_block.cuh"), "contract_tc_kernel": ("contract_tc.cu",),
             "epilogue_tc_kernel": ("epilogue_tc.cu", "tile_ops.cuh")}[kernel]
    h = hashlib.sha256()
    for f in files + ("common.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "pair_representation_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, N: int):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json),
    or None when there is none for this kernel at this N or the kernel's source
    has changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rows = json.load(f)
    for r in rows.get("kernels", []):
        if r.get("kernel") == kernel and r.get("N") == N and r.get("src_sha") == source_sha(kernel):
            return int(r["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------- multi-rank host logic

def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest value over all ranks (timing is the slowest replica's)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def pair_cells_per_s(world: int, steps: int, n_dirs: int, N: int, total_ms: float) -> float:
    """Whole-job throughput: every rank processes steps * n_dirs * N^2 pair-cells."""
    return world * steps * n_dirs * N * N / (total_ms / 1e3)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a background thread."""

    BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.nvml = None
            self.err = str(e)
        self.period = period_s

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                r = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.BITS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.nvml:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.nvml:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- oracle (CPU baseline)

def oracle_sample(workload, n_idx: int, seed: int = 0, threads=None):
    """Run the oracle on the sampled grid I x I (|I| = n_idx) in every direction of the
    workload; returns (cells computed, seconds)."""
    import numpy as np

    import oracle
    import pair_inputs as pi
    rng = np.random.default_rng([workload.seed, 77, seed])
    I = np.sort(rng.choice(workload.N, size=min(n_idx, workload.N), replace=False)).astype(np.int32)
    case = pi.make_workload(workload)
    t0 = time.perf_counter()
    cells = 0
    for d in workload.directions:
        oracle.trimul_grid(case, d, I, threads=threads)
        cells += len(I) ** 2
    return cells, time.perf_counter() - t0


def calibrated_oracle(workload, budget_s: float, threads=None):
    """Choose |I| so the oracle sample takes about budget_s seconds, then run it."""
    cells, t = oracle_sample(workload, 8, seed=1, threads=threads)
    per_line = t / 8.0  # projection cost is linear in |I| and dominates
    n_idx = int(max(8, min(workload.N, budget_s / max(per_line, 1e-6))))
    cells, t = oracle_sample(workload, n_idx, threads=threads)
    return cells, t, n_idx


# ---------------------------------------------------------------- GPU arm

def per_config_timings(tm, pi, torch, dev, stream, warmup=3, reps=5):
    """Secondary figures: every workload and each direction separately, one
    trimul_forward call per timing (CUDA events), L2 flushed before each call
    (median and best), plus the median with a warm L2 (calls back to back)."""
    res = {}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for wid, w in sorted(pi.WORKLOADS.items()):
        case = pi.make_workload(w)
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        z = torch.from_numpy(case["z"]).to(dev).to(tdt)
        mask = torch.from_numpy(case["mask"]).to(dev).to(tdt)
        del case["z"]
        out = torch.empty_like(z)
        entry = {"N": w.N, "dtype": w.dtype}
        for d in w.directions:
            cls = tm.TriangleMultiplicationOutgoing if d == "outgoing" else tm.TriangleMultiplicationIncoming
            sd = {key: torch.from_numpy(case[field]) for field, key, _ in tm.STATE_KEYS if field in case}
            layer = cls(128, 128).load_state_dict(sd).to(dev, tdt)
            for _ in range(warmup):
                layer(z, mask, out=out, stream=stream)
            cold, warm = [], []
            for _ in range(reps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                layer(z, mask, out=out, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize()
                cold.append(e0.elapsed_time(e1) * 1e3)
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                layer(z, mask, out=out, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize()
                warm.append(e0.elapsed_time(e1) * 1e3)
            cold.sort()
            warm.sort()
            med = cold[len(cold) // 2]
            entry[d] = {"median_us": round(med, 1), "best_us": round(cold[0], 1),
                        "warm_l2_median_us": round(warm[len(warm) // 2], 1),
                        "pair_cells_per_s": round(w.N * w.N / (med * 1e-6)),
                        "tflops": round(w.N * w.N * flops_per_cell(w.N) / (med * 1e-6) / 1e12, 1)}
            del layer
        res[w.name] = entry
        del z, mask, out
        torch.cuda.empty_cache()
    return res


def backward_flops_per_cell(N: int) -> int:
    """GEMM FLOP per cell of one trimul_backward call: the recomputed a, b and x
    (4 projections + contraction), then P (5 projections), Y, dL/dxh, the
    contraction's adjoint (2 products), the 6 weight gradients and dL/dzh (5)."""
    g = 2 * 128 * 128
    return 4 * g + 256 * N + 5 * g + g + g + 2 * 256 * N + 6 * g + 5 * g


# HBM bytes per cell that the backward's steps move at their minimum (each
# array read or written once per step that uses it), excluding the recomputed
# forward: LayerNorms 2 x 520, P 1536, Y 512, gate 1280, dL/dxh 768, LN_out
# adjoint 1032, contraction adjoint 1536, input-gate adjoint 2562, weight
# gradients 2048, dL/dzh 1792, LN_in adjoint 1032.
BACKWARD_BYTES_PER_CELL = 2 * 520 + 1536 + 512 + 1280 + 768 + 1032 + 1536 + 2562 + 2048 + 1792 + 1032


def backward_timings(tm, pi, torch, dev, stream, peaks, warmup=3, reps=7):
    """Secondary figure: one trimul_backward call per direction on the N = 768
    workload (dout drawn N(0, 1), bf16), CUDA events, L2 flushed before each call."""
    import numpy as np
    w = pi.WORKLOADS[DEFAULT_WORKLOAD]
    N = w.N
    case = pi.make_workload(w)
    z = torch.from_numpy(case["z"]).to(dev).to(torch.bfloat16)
    mask = torch.from_numpy(case["mask"]).to(dev).to(torch.bfloat16)
    dout = torch.from_numpy(np.random.default_rng([7, 8]).standard_normal((N, N, 128), dtype=np.float32)).to(dev)
    dout = dout.to(torch.bfloat16)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    res = {"workload": w.name, "N": N, "dtype": "bf16", "gemm_flop_per_cell": backward_flops_per_cell(N),
           "hbm_bytes_per_cell_min": BACKWARD_BYTES_PER_CELL,
           "recompute": "a, b, x recomputed by the forward kernels inside the call"}
    for d, cls in (("outgoing", tm.TriangleMultiplicationOutgoing), ("incoming", tm.TriangleMultiplicationIncoming)):
        sd = {key: torch.from_numpy(case[field]) for field, key, _ in tm.STATE_KEYS if field in case}
        layer = cls(128, 128).load_state_dict(sd).to(dev, torch.bfloat16)
        for _ in range(warmup):
            layer.backward(z, dout, mask, stream=stream)
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            layer.backward(z, dout, mask, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        ts.sort()
        med = ts[len(ts) // 2]
        res[d] = {"median_us": round(med, 1), "best_us": round(ts[0], 1),
                  "pair_cells_per_s": round(N * N / (med * 1e-6)),
                  "gemm_tflops": round(N * N * backward_flops_per_cell(N) / (med * 1e-6) / 1e12, 1),
                  "min_bytes_gbs": round(N * N * BACKWARD_BYTES_PER_CELL / (med * 1e-6) / 1e9, 1)}
        # The same call right after a forward on the same inputs, reusing its a, b and x.
        layer(z, mask, stream=stream)
        tr = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            layer.backward(z, dout, mask, stream=stream, reuse_forward=True)
            e1.record(stream)
            torch.cuda.synchronize()
            tr.append(e0.elapsed_time(e1) * 1e3)
        tr.sort()
        res[d]["reuse_forward_median_us"] = round(tr[len(tr) // 2], 1)
        del layer
    res["hbm_peak_gbs"] = peaks["hbm_gbs"]
    del z, mask, dout, flush
    torch.cuda.empty_cache()
    return res


ATTN_SHAPE = {"batch": 8, "n_atoms": 768 * 24, "heads": 4, "head_dim": 32}


def attention_inputs(B, n, H, seed=5):
    """Synthetic q, k, v, bias ~ N(0, 1) and an atom mask with a padded tail (5 %), as bf16-valued numpy."""
    import numpy as np
    rng = np.random.default_rng([seed, 31])
    q, k, v = (rng.standard_normal((B, n, H, 32), dtype=np.float32) for _ in range(3))
    bias = rng.standard_normal((B, (n + 31) // 32, H, 32, 128), dtype=np.float32)
    mask = np.ones((B, n), dtype=np.float32)
    mask[:, n - n // 20:] = 0
    return q, k, v, bias, mask


def attention_timings(tm, torch, dev, stream, peaks, warmup=3, reps=10):
    """Secondary figure: windowed atom attention (atomattn_forward) on 8 x 18432 atoms
    (a 768-token crop at 24 atoms per token, 8 samples), 4 heads of 32, with bias and
    mask; CUDA events, L2 flushed before each call; the float64 oracle timed on
    batch element 0 (all its windows and heads)."""
    import numpy as np
    from oracle.atomattn import atom_attention as oracle_attention
    B, n, H = ATTN_SHAPE["batch"], ATTN_SHAPE["n_atoms"], ATTN_SHAPE["heads"]
    arrs = attention_inputs(B, n, H)
    t = [torch.from_numpy(a).to(dev).to(torch.bfloat16) for a in arrs]
    q, k, v, bias, mask = t
    out = torch.empty_like(q)
    ws = torch.zeros(tm.atomattn_workspace_size(), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        tm.atom_attention(q, k, v, bias, mask, out=out, workspace=ws, stream=stream)
    ts = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        tm.atom_attention(q, k, v, bias, mask, out=out, workspace=ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    ts.sort()
    med = ts[len(ts) // 2]
    W = (n + 31) // 32
    # Minimum HBM bytes: q, k, v read and out written once, bias and mask read once.
    min_bytes = 4 * B * n * H * 32 * 2 + B * W * H * 32 * 128 * 2 + B * n * 2
    flops = B * W * H * 2 * (32 * 128 * 32 * 2)  # S = Q K^T and O = P V per window
    # Oracle on a bounded sample: batch element 0.
    na = n
    sample = [a[:1] for a in arrs]
    t0 = time.perf_counter()
    oracle_attention(*[np.asarray(x, dtype=np.float64) for x in sample])
    osec = time.perf_counter() - t0
    res = {"shape": dict(ATTN_SHAPE, bias=True, atom_mask="last 5 % padded"), "dtype": "bf16",
           "median_us": round(med, 1), "best_us": round(ts[0], 1),
           "atoms_per_s": round(B * n / (med * 1e-6)),
           "min_bytes": min_bytes, "min_bytes_gbs": round(min_bytes / (med * 1e-6) / 1e9, 1),
           "frac_of_hbm_peak": round(min_bytes / (med * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
           "tflops": round(flops / (med * 1e-6) / 1e12, 1),
           "cpu_oracle": {"atoms_per_s": round(na / osec), "sample": f"{na} atoms x {H} heads of batch element 0",
                          "kind": "oracle", "seconds": round(osec, 2)}}
    del q, k, v, bias, mask, out, flush
    torch.cuda.empty_cache()
    return res


def mxfp8_timings(tm, pi, torch, dev, stream, peaks, wids=(3, 4, 5), warmup=3, reps=5):
    """Secondary figure: the MXFP8 contraction (trimul_contract_mxfp8: quantizer and
    block-scaled MMA kernel) beside the bf16 one (trimul_contract) on the same a, b
    (written by the prologue), per workload and direction, CUDA events, L2 flushed
    before each call; and the whole MXFP8 layer (trimul_forward_mxfp8, which
    quantizes inside the prologue) beside the bf16 layer (trimul_forward)."""
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    code = {"outgoing": tm.OUTGOING, "incoming": tm.INCOMING}

    def timed(fn):
        for _ in range(warmup):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        ts.sort()
        return ts[len(ts) // 2]

    res = {"format": "E4M3 elements, E8M0 scale per 32 along k (OCP MX v1.0); fp32 accumulation; x in bf16"}
    for wid in wids:
        w = pi.WORKLOADS[wid]
        case = pi.make_workload(w)
        z = torch.from_numpy(case["z"]).to(dev).to(torch.bfloat16)
        mask = torch.from_numpy(case["mask"]).to(dev).to(torch.bfloat16)
        del case["z"]
        sd = {key: torch.from_numpy(case[field]) for field, key, _ in tm.STATE_KEYS if field in case}
        layer = tm.TriangleMultiplicationOutgoing(128, 128).load_state_dict(sd).to(dev, torch.bfloat16)
        p = layer.params(w.N)
        ws = torch.empty(tm.trimul_workspace_size_mxfp8(w.N, 128, 128), dtype=torch.uint8, device=dev)
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
        tm.trimul_prologue(z, mask, p, stream)
        flop = 2 * w.N ** 3 * 128
        entry = {"N": w.N}
        for d in w.directions:
            t_mx = timed(lambda: tm.trimul_contract_mxfp8(p, code[d], stream))
            t_bf = timed(lambda: tm.trimul_contract(p, code[d], stream))
            # The MMA kernel alone, on the operands the quantizer just wrote.
            t_mma = timed(lambda: tm.trimul_mma_mxfp8(p, stream))
            t_pro_mx = timed(lambda: tm.trimul_prologue_mxfp8(z, mask, p, code[d], stream))
            t_pro = timed(lambda: tm.trimul_prologue(z, mask, p, stream))
            entry[d] = {"mxfp8_us": round(t_mx, 1), "bf16_us": round(t_bf, 1),
                        "mxfp8_tflops": round(flop / (t_mx * 1e-6) / 1e12, 1),
                        "bf16_tflops": round(flop / (t_bf * 1e-6) / 1e12, 1),
                        "speedup": round(t_bf / t_mx, 3),
                        "mma_us": round(t_mma, 1), "mma_tflops": round(flop / (t_mma * 1e-6) / 1e12, 1),
                        "mma_speedup": round(t_bf / t_mma, 3),
                        "prologue_mxfp8_us": round(t_pro_mx, 1), "prologue_bf16_us": round(t_pro, 1)}
        out = torch.empty_like(z)
        for d in w.directions:
            t = timed(lambda: tm.trimul_forward_mxfp8(z, mask, p, code[d], out, stream))
            t_bf = timed(lambda: tm.trimul_forward(z, mask, p, code[d], out, stream))
            entry[d]["layer_us"] = round(t, 1)
            entry[d]["layer_bf16_us"] = round(t_bf, 1)
            entry[d]["layer_speedup"] = round(t_bf / t, 3)
            entry[d]["layer_pair_cells_per_s"] = round(w.N * w.N / (t * 1e-6))
        res[w.name] = entry
        rc, detail = tm.trimul_device_status(p, stream)
        if rc != 0:
            raise RuntimeError(f"device status {rc} {detail}")
        del z, mask, ws, layer
        torch.cuda.empty_cache()
    return res


def run_mxfp8_only(args):
    """--mxfp8-only: the MXFP8 secondary figure alone, on one GPU."""
    import torch

    import pair_inputs as pi
    import pair_representation_b200 as tm
    from pair_representation_b200 import build as tmbuild

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    tmbuild.build()
    tm.lib()
    peaks, _ = load_peaks()
    wids = tuple(int(x) for x in args.mx_workloads.split(","))
    res = mxfp8_timings(tm, pi, torch, dev, torch.cuda.current_stream(dev), peaks, wids=wids, warmup=args.warmup,
                        reps=args.steps)
    print(json.dumps({"mxfp8": res}), flush=True)


def run_attention_only(args):
    """--attention-only: the atom-attention secondary figure alone, on one GPU."""
    import torch

    import pair_representation_b200 as tm
    from pair_representation_b200 import build as tmbuild

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    tmbuild.build()
    tm.lib()
    peaks, _ = load_peaks()
    res = attention_timings(tm, torch, dev, torch.cuda.current_stream(dev), peaks, args.warmup, args.steps)
    print(json.dumps({"atom_attention": res}), flush=True)


def backward_blocked_timing(tm, pi, torch, dev, stream, block_rows=256, warmup=1, reps=2):
    """The backward of the largest workload (N = 3605, outgoing) in blocks of
    `block_rows` rows: the workspace that trimul_backward_workspace_size_rows
    gives for them against the whole-grid size, and the time per call (CUDA
    events). dout is drawn on the device (values do not change the work)."""
    w = pi.WORKLOADS[5]
    N = w.N
    case = pi.make_workload(w)
    z = torch.from_numpy(case["z"]).to(dev).to(torch.bfloat16)
    mask = torch.from_numpy(case["mask"]).to(dev).to(torch.bfloat16)
    del case["z"]
    gen = torch.Generator(device=dev).manual_seed(11)
    dout = torch.randn(z.shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    sd = {key: torch.from_numpy(case[field]) for field, key, _ in tm.STATE_KEYS if field in case}
    layer = tm.TriangleMultiplicationOutgoing(128, 128).load_state_dict(sd).to(dev, torch.bfloat16)
    for _ in range(warmup):
        layer.backward(z, dout, mask, stream=stream, block_rows=block_rows)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer.backward(z, dout, mask, stream=stream, block_rows=block_rows)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    ts.sort()
    med = ts[len(ts) // 2]
    res = {"workload": w.name, "N": N, "direction": "outgoing", "block_rows": block_rows,
           "workspace_gb": round(tm.trimul_backward_workspace_size_rows(N, block_rows) / 1e9, 2),
           "whole_grid_workspace_gb": round(tm.trimul_backward_workspace_size(N) / 1e9, 2),
           "median_us": round(med, 1), "pair_cells_per_s": round(N * N / (med * 1e-6)),
           "gemm_tflops": round(N * N * backward_flops_per_cell(N) / (med * 1e-6) / 1e12, 1)}
    del layer, z, mask, dout
    torch.cuda.empty_cache()
    return res


def run_backward_only(args):
    """--backward-only: the backward secondary figure alone, on one GPU."""
    import torch

    import pair_inputs as pi
    import pair_representation_b200 as tm
    from pair_representation_b200 import build as tmbuild

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    tmbuild.build()
    tm.lib()
    peaks, _ = load_peaks()
    res = backward_timings(tm, pi, torch, dev, torch.cuda.current_stream(dev), peaks, args.warmup, args.steps)
    if args.backward_blocked:
        res["blocked_large"] = backward_blocked_timing(tm, pi, torch, dev, torch.cuda.current_stream(dev))
    print(json.dumps({"backward": res}), flush=True)


def run_sharded(args, rank, world, local_rank):
    """--mode sharded: one layer split over the ranks (row blocks for the prologue and
    epilogue, channel blocks for the contraction, NCCL send/recv between them;
    pair_representation_b200.sharded). Total work is fixed as the rank count grows
    ("scaling": "strong"): value = steps x directions x N^2 / the slowest rank's time."""
    import torch

    import pair_inputs as pi
    import pair_representation_b200 as tm
    from pair_representation_b200 import build as tmbuild
    from pair_representation_b200.sharded import CudaStages, ShardedTriangleMultiplication, ShardPlan

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    if rank == 0:
        tmbuild.build()
    if world > 1:
        dist.barrier()
    tm.lib()
    w = pi.WORKLOADS[args.workload]
    N = w.N
    plan = ShardPlan(N, world)
    r0, r1 = plan.rows(rank)
    z_rows = torch.from_numpy(pi.draw_z(N, 128, w.seed, w.channel_scale, True, rows=range(r0, r1))).to(dev)
    z_rows = z_rows.to(torch.bfloat16)
    m = pi.residue_mask(N, w.n_valid)
    mask_rows = torch.from_numpy(pi.pair_mask(m)[r0:r1].copy()).to(dev).to(torch.bfloat16)
    case = pi.make_workload(w, with_z=False)
    sd = {key: torch.from_numpy(case[field]) for field, key, _ in tm.STATE_KEYS if field in case}
    layer = tm.TriangleMultiplicationOutgoing(128, 128).load_state_dict(sd).to(dev, torch.bfloat16)
    p = layer.params(N)
    ws = torch.zeros(tm.trimul_shard_workspace_size(N, r1 - r0), dtype=torch.uint8, device=dev)
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    code = {"outgoing": tm.OUTGOING, "incoming": tm.INCOMING}
    layers = {d: ShardedTriangleMultiplication(plan, rank, code[d], CudaStages(tm, p), dev, torch.bfloat16, dist)
              for d in w.directions}
    outs = {d: torch.empty_like(z_rows) for d in w.directions}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        for d in w.directions:
            layers[d](z_rows, mask_rows, outs[d])

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    rc, detail = tm.trimul_device_status(p)
    if rc != 0:
        raise RuntimeError(f"device status {rc} {detail}")
    total_ms = 0.0
    sampler = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for _ in range(args.steps):
        flush.zero_()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        total_ms += e0.elapsed_time(e1)
    sampler.stop()
    total_ms = max_over_ranks(total_ms, dist if world > 1 else None, dev)
    value = args.steps * len(w.directions) * N * N / (total_ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "N": N, "c_z": 128, "c_h": 128, "batch": 1,
                       "directions": list(w.directions),
                       "l2": "flushed (512 MB write) before every step, outside the timed events",
                       "parallelism": f"sharded x{world}: row blocks (prologue, epilogue), channel blocks "
                                      f"(contraction), NCCL send/recv exchanges"},
            "gpu_launches": args.steps * len(w.directions) * 3, "clocks": sampler.summary()}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import pair_inputs as pi
    import pair_representation_b200 as tm
    from pair_representation_b200 import build as tmbuild

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    if rank == 0:
        tmbuild.build()
    if dist:
        dist.barrier()
    tm.lib()

    w = pi.WORKLOADS[args.workload]
    N = w.N
    case = pi.make_workload(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    z_host = torch.from_numpy(case["z"]).to(tdt).pin_memory()
    m_host = torch.from_numpy(case["mask"]).to(tdt).pin_memory()
    z = z_host.to(dev)
    mask = m_host.to(dev)
    layers = {}
    for name, cls in (("outgoing", tm.TriangleMultiplicationOutgoing), ("incoming", tm.TriangleMultiplicationIncoming)):
        sd = {key: torch.from_numpy(case[field]) for field, key, _ in tm.STATE_KEYS if field in case}
        layers[name] = cls(128, 128).load_state_dict(sd).to(dev, tdt)
    dirs = list(w.directions)
    code = {"outgoing": tm.OUTGOING, "incoming": tm.INCOMING}
    params = {d: layers[d].params(N) for d in dirs}
    outs = {d: torch.empty_like(z) for d in dirs}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    names = ("prologue_tc_kernel", "contract_tc_kernel", "epilogue_tc_kernel") if w.dtype == "bf16" else \
        ("prologue_f32_kernel", "contract_f32_kernel", "epilogue_f32_kernel")

    def one_step(evs, sh):
        """One step: both directions, each as its three stage calls on stream `sh`. With `evs`
        (a list), a timing event is recorded before every kernel and after the last."""
        cur = torch.cuda.current_stream(dev)

        def mark():
            if evs is not None:
                evs.append(torch.cuda.Event(enable_timing=True, external=True))
                evs[-1].record(cur)
        for d in dirs:
            p = params[d]
            mark()
            tm.trimul_prologue(z, mask, p, sh)
            mark()
            tm.trimul_contract(p, code[d], sh)
            mark()
            tm.trimul_epilogue(z, p, outs[d], sh)
        mark()

    for _ in range(args.warmup):
        flush.zero_()
        one_step(None, sh)
    torch.cuda.synchronize()
    for d in dirs:
        rc, detail = tm.trimul_device_status(params[d], sh)
        if rc != 0:
            raise RuntimeError(f"device status {rc} {detail}")

    # The step runs as a CUDA graph of its six stage calls (captured once; the host-side
    # argument checks and tensor-map encoding happen at capture), which shortens the gap
    # between dependent kernels from about 2 us to under 1 us. The timed K steps replay it
    # between step-boundary events; a second graph, with a timing event before every kernel
    # and after the last, gives the per-kernel breakdown and the roofline in a second pass of
    # K steps. The same step launched eagerly is timed as well (`eager_ms_per_step`).
    cap = torch.cuda.Stream(dev)
    graph, graph_ev, evs_cap = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), []
    with torch.cuda.graph(graph, stream=cap, capture_error_mode="relaxed"):
        one_step(None, cap.cuda_stream)
    with torch.cuda.graph(graph_ev, stream=cap, capture_error_mode="relaxed"):
        one_step(evs_cap, cap.cuda_stream)
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        graph.replay()
        graph_ev.replay()
    torch.cuda.synchronize()
    for d in dirs:
        rc, detail = tm.trimul_device_status(params[d], sh)
        if rc != 0:
            raise RuntimeError(f"device status {rc} {detail}")

    sampler = ClockSampler(local_rank)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    step_ms = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        step_ms.append((e0, e1))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    step_ms = [e0.elapsed_time(e1) for e0, e1 in step_ms]
    total_ms = sum(step_ms)
    kern_ms = {n: 0.0 for n in names}
    for _ in range(args.steps):
        flush.zero_()
        graph_ev.replay()
        torch.cuda.synchronize()
        for k, d in enumerate(dirs):
            for s_, n in enumerate(names):
                kern_ms[n] += evs_cap[3 * k + s_].elapsed_time(evs_cap[3 * k + s_ + 1])
    eager_ms = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        one_step(None, sh)
        e1.record(stream)
        eager_ms.append((e0, e1))
    torch.cuda.synchronize()
    sampler.stop()
    eager_ms_per_step = sum(e0.elapsed_time(e1) for e0, e1 in eager_ms) / args.steps
    del graph, graph_ev
    launches = {n: args.steps * len(dirs) for n in names}
    total_ms = max_over_ranks(total_ms, dist, dev)

    # ---- end to end through the public layer API, host buffers in and out
    # Every step copies its inputs (z, mask) from pinned host memory and both outputs back,
    # inside the timed region. Steps are pipelined over three streams with two device slots:
    # step i's host-to-device copy, step i - 1's layer calls and step i - 2's device-to-host
    # copy can run at once (the copy engines work in both directions at the same time). The
    # same steps run one at a time, each synchronised, are reported as `serial_value`.
    e2e = None
    if not args.no_e2e:
        slots = [{"z": torch.empty_like(z), "m": torch.empty_like(mask),
                  "o": {d: torch.empty_like(z) for d in dirs},
                  "h": {d: torch.empty(z.shape, dtype=tdt, pin_memory=True) for d in dirs}} for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(k):
            ev_comp, ev_out = [None] * k, [None] * k
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(s_in)
            for i in range(k):
                sl = slots[i & 1]
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])  # the slot's z and mask have been read
                with torch.cuda.stream(s_in):
                    sl["z"].copy_(z_host, non_blocking=True)
                    sl["m"].copy_(m_host, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
                stream.wait_event(ev_in)
                if i >= 2:
                    stream.wait_event(ev_out[i - 2])  # the slot's outputs have been copied out
                for d in dirs:
                    layers[d](sl["z"], sl["m"], out=sl["o"][d], stream=stream)
                ev_comp[i] = torch.cuda.Event()
                ev_comp[i].record(stream)
                s_out.wait_event(ev_comp[i])
                with torch.cuda.stream(s_out):
                    for d in dirs:
                        sl["h"][d].copy_(sl["o"][d], non_blocking=True)
                ev_out[i] = torch.cuda.Event()
                ev_out[i].record(s_out)
            s_out.wait_event(ev_out[k - 1])
            t1.record(s_out)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1)

        e2e_run(max(args.warmup, 2))
        if dist:
            dist.barrier()
        e2e_ms = max_over_ranks(e2e_run(args.steps), dist, dev)

        out_host = slots[0]["h"]
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def e2e_step():
            zd = z_host.to(dev, non_blocking=True)
            md = m_host.to(dev, non_blocking=True)
            for d in dirs:
                o = layers[d](zd, md, out=outs[d], stream=stream)
                out_host[d].copy_(o, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        serial_ms = 0.0
        for _ in range(args.steps):
            flush.zero_()
            ev0.record(stream)
            e2e_step()
            ev1.record(stream)
            torch.cuda.synchronize()
            serial_ms += ev0.elapsed_time(ev1)
        serial_ms = max_over_ranks(serial_ms, dist, dev)
        e2e = {"value": pair_cells_per_s(world, args.steps, len(dirs), N, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": z_host.numel() * z_host.element_size() + m_host.numel() * m_host.element_size(),
               "d2h_bytes_per_step": sum(out_host[d].numel() * out_host[d].element_size() for d in dirs),
               "pipelined": "copy-in, layer and copy-out streams, two device slots",
               "serial_value": pair_cells_per_s(world, args.steps, len(dirs), N, serial_ms)}
        del slots

    # ---- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    alg = kernel_algorithmic(N)
    dom = max(kern_ms, key=lambda n: kern_ms[n])
    per_launch_s = kern_ms[dom] / launches[dom] / 1e3
    breakdown = {}
    for n in names:
        avg = kern_ms[n] / launches[n] / 1e3
        entry = {"avg_us": round(avg * 1e6, 2), "share": round(kern_ms[n] / sum(kern_ms.values()), 4)}
        if n in alg:
            q, u, bound = alg[n]
            if u == "bytes":
                entry["achieved_gbs"] = round(q / avg / 1e9, 1)
                entry["frac_hbm"] = round(q / avg / 1e9 / peaks["hbm_gbs"], 4)
                entry["frac_hbm_nominal"] = round(q / avg / 1e9 / NOMINAL_PEAKS["hbm_gbs"], 4)
            else:
                entry["achieved_tflops"] = round(q / avg / 1e12, 1)
                entry["frac_tensor"] = round(q / avg / 1e12 / peaks["bf16_tflops"], 4)
                entry["frac_tensor_nominal"] = round(q / avg / 1e12 / NOMINAL_PEAKS["bf16_tflops"], 4)
        breakdown[n] = entry
    roofline = None
    if dom in alg:
        q, u, bound = alg[dom]
        if u == "bytes":
            achieved, peak, unit = q / per_launch_s / 1e9, peaks["hbm_gbs"], "GB/s"
        else:
            achieved, peak, unit = q / per_launch_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        roofline = {"kernel": dom, "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                    "frac": round(achieved / peak, 4), "traffic": ncu_traffic(dom, N),
                    "peak_source": f"{peak_src} ({'burst' if u != 'bytes' else 'copy'})"}

    # ---- CPU baseline: the oracle on a bounded sample, rank 0 only, N = 1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cells, secs, n_idx = calibrated_oracle(w, args.oracle_seconds)
        cpu = {"value": cells / secs, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
               "sample": f"float64 oracle (grid mode) on {n_idx} x {n_idx} sampled cells of the N={N} "
                         f"workload, {'+'.join(dirs)}: {cells} pair-cells in {secs:.1f} s"}

    value = pair_cells_per_s(world, args.steps, len(dirs), N, total_ms)
    tflops = world * args.steps * len(dirs) * N * N * flops_per_cell(N) / (total_ms / 1e3) / 1e12
    clocks = sampler.summary()
    configs = None
    backward = None
    if rank == 0 and world == 1 and not args.no_configs:
        del flush
        configs = per_config_timings(tm, pi, torch, dev, stream)
        if not args.no_cpu_baseline:
            # The float64 oracle on every workload: the whole layer where it takes seconds
            # (N <= 384), a sampled grid of about 2 s elsewhere, with the full layer's time
            # extrapolated from the measured rate (every cell costs the same).
            for wid, wk in sorted(pi.WORKLOADS.items()):
                if wk.name not in configs:
                    continue
                if wk.N <= 384:
                    cells, secs = oracle_sample(wk, wk.N)
                    sample, n_idx = "the whole layer", wk.N
                else:
                    cells, secs, n_idx = calibrated_oracle(wk, 2.0)
                    sample = f"{n_idx} x {n_idx} sampled cells per direction"
                rate = cells / secs
                configs[wk.name]["cpu_oracle"] = {
                    "pair_cells_per_s": round(rate, 1), "sample": sample, "cores": os.cpu_count(),
                    "full_layer_s": round(wk.N * wk.N * len(wk.directions) / rate, 2),
                    "full_layer_s_is": "measured" if n_idx == wk.N else "extrapolated"}
    if rank == 0 and world == 1 and not args.no_backward:
        backward = backward_timings(tm, pi, torch, dev, stream, peaks)
    attention = None
    if rank == 0 and world == 1 and not args.no_attention:
        attention = attention_timings(tm, torch, dev, stream, peaks)
    mxfp8 = None
    if rank == 0 and world == 1 and not args.no_mxfp8:
        mxfp8 = mxfp8_timings(tm, pi, torch, dev, stream, peaks)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "N": N, "c_z": 128, "c_h": 128, "batch": 1, "directions": dirs,
                   "l2": "flushed (512 MB write) before every step, outside the timed events",
                   "launch": "CUDA graph of the step's six stage calls, replayed",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "eager_ms_per_step": round(eager_ms_per_step, 4),
        "tflops": round(tflops, 2),
        "tflops_frac_of_bf16_peak": round(tflops / peaks["bf16_tflops"], 4),
        "roofline": roofline,
        "kernels": breakdown,
        "peaks": {"frac_hbm and frac_tensor against": dict(peaks, source=peak_src),
                  "frac_*_nominal against (datasheet)": NOMINAL_PEAKS},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": sum(launches.values()),
        "clocks": clocks,
        "per_config": configs,
        "backward": backward,
        "atom_attention": attention,
        "mxfp8": mxfp8,
    }
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The float64 oracle as it stands, on the host cores, on bounded samples of the workload."""
    if rank != 0:
        return
    import pair_inputs as pi
    w = pi.WORKLOADS[args.workload]
    per_step = max(1.0, args.reference_budget / max(1, args.steps + args.warmup))
    cells, t = 0, 0.0
    _, _, n_idx = calibrated_oracle(w, per_step)
    for k in range(args.warmup):
        oracle_sample(w, n_idx, seed=100 + k)
    for k in range(args.steps):
        c, s = oracle_sample(w, n_idx, seed=k)
        cells += c
        t += s
    value = cells / t
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "N": w.N, "c_z": 128, "c_h": 128, "batch": 1,
                   "directions": list(w.directions)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"each step: float64 oracle (grid mode) on {n_idx} x {n_idx} sampled cells "
                                   f"of the N={w.N} workload, {'+'.join(w.directions)}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--mode", choices=("replicas", "sharded"), default="replicas",
                    help="replicas: every rank runs the whole layer (default); sharded: one layer split "
                         "over the ranks")
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=(1, 2, 3, 4, 5))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload secondary timings")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward secondary timing")
    ap.add_argument("--backward-blocked", action="store_true",
                    help="with --backward-only: also the N = 3605 backward in blocks of 256 rows")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only trimul_backward (W warm-up and K timed calls per direction) and print that")
    ap.add_argument("--no-attention", action="store_true", help="skip the atom-attention secondary timing")
    ap.add_argument("--attention-only", action="store_true",
                    help="time only atomattn_forward (W warm-up and K timed calls) and print that")
    ap.add_argument("--no-mxfp8", action="store_true", help="skip the MXFP8 secondary timing")
    ap.add_argument("--mxfp8-only", action="store_true",
                    help="time only the MXFP8 contraction beside the bf16 one and print that")
    ap.add_argument("--mx-workloads", default="3,4,5",
                    help="workload ids --mxfp8-only runs (3: N = 768, 4: N = 2048, 5: N = 3605)")
    ap.add_argument("--oracle-seconds", type=float, default=15.0)
    ap.add_argument("--reference-budget", type=float, default=120.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.backward_only:
        run_backward_only(args)
    elif args.attention_only:
        run_attention_only(args)
    elif args.mxfp8_only:
        run_mxfp8_only(args)
    elif args.mode == "sharded":
        run_sharded(args, rank, world, local_rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
